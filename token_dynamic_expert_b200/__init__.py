"""B200-native (sm_100a) ACE per-token expert skipping for routed SwiGLU MoE
layers: a C-ABI library (``libace.so``, ``include/ace.h``) and its thin
Python binding :mod:`token_dynamic_expert_b200.ace`.

Importing the binding loads ``libace.so`` and raises if it is not built; the
package has no CPU or eager fallback.
"""
__all__ = ["ace", "build"]
