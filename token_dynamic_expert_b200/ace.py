"""ctypes binding of libace (``include/ace.h``), with the C names.

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the computation runs in libace's kernels.
There is no fallback: if ``libace.so`` is missing or fails to load, importing
this module raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libace.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libace.so not built: run `python -m token_dynamic_expert_b200.build` "
                      "(expected at %s)" % LIB_PATH)
_lib = ctypes.CDLL(LIB_PATH)

# ------------------------------------------------------------------ C types
ACE_OK, ACE_ERR_INVALID_ARG, ACE_ERR_WORKSPACE, ACE_ERR_CUDA, ACE_ERR_UNSUPPORTED, \
    ACE_ERR_DEVICE_FAULT, ACE_ERR_TIMEOUT, ACE_ERR_IO = range(8)
ACE_BF16, ACE_F32 = 0, 1
ACE_GSP_FRO, ACE_GSP_SPECTRAL = 0, 1
ACE_FUSE_MAX, ACE_FUSE_MIN, ACE_FUSE_MEAN, ACE_FUSE_GSP, ACE_FUSE_RCR = 0, 1, 2, 3, 4
FUSIONS = {"max": ACE_FUSE_MAX, "min": ACE_FUSE_MIN, "mean": ACE_FUSE_MEAN, "gsp": ACE_FUSE_GSP,
           "rcr": ACE_FUSE_RCR}
ACE_FLAG_BAD_INDEX, ACE_FLAG_TIMEOUT, ACE_FLAG_OVERFLOW = 0x1, 0x2, 0x4

_vp = ctypes.c_void_p


class ace_layer(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("E", ctypes.c_int), ("m", ctypes.c_int), ("k", ctypes.c_int),
                ("dtype", ctypes.c_int), ("gamma", _vp), ("w_router", _vp), ("router_bias", _vp),
                ("w_gate", _vp), ("w_up", _vp), ("w_down", _vp), ("amax", _vp), ("a_gsp", _vp),
                ("a_rcr", _vp)]


class ace_fwd_opts(ctypes.Structure):
    _fields_ = [("tau", ctypes.c_float), ("renorm_topk", ctypes.c_int), ("fusion", ctypes.c_int),
                ("eps_rms", ctypes.c_float)]


class ace_debug_out(ctypes.Structure):
    _fields_ = [("topk_idx", _vp), ("gate", _vp), ("score", _vp), ("keep", _vp),
                ("expert_offsets", _vp), ("slot_token", _vp), ("slot_rank", _vp),
                ("n_kept", _vp), ("logits", _vp), ("ev_experts_begin", _vp),
                ("ev_experts_mid", _vp), ("ev_experts_end", _vp), ("trace", _vp)]


class ace_table_opts(ctypes.Structure):
    _fields_ = [("gsp_norm", ctypes.c_int), ("eps", ctypes.c_float), ("rho", ctypes.c_float),
                ("power_iters", ctypes.c_int)]


_P = ctypes.POINTER
_lib.ace_workspace_size.argtypes = [_P(ace_layer), ctypes.c_int]
_lib.ace_workspace_size.restype = ctypes.c_size_t
_lib.ace_moe_forward.argtypes = [_P(ace_layer), _vp, ctypes.c_int, _P(ace_fwd_opts), _vp, _vp,
                                 ctypes.c_size_t, _P(ace_debug_out), _vp]
_lib.ace_moe_forward.restype = ctypes.c_int
_lib.ace_moe_scores.argtypes = [_P(ace_layer), _vp, ctypes.c_int, _P(ace_fwd_opts), _vp, _vp, _vp,
                                ctypes.c_size_t, _vp]
_lib.ace_moe_scores.restype = ctypes.c_int
_lib.ace_moe_route.argtypes = [_P(ace_layer), _vp, ctypes.c_int, _P(ace_fwd_opts), _vp, _vp, _vp,
                               _vp, _vp, ctypes.c_size_t, _vp]
_lib.ace_moe_route.restype = ctypes.c_int
_lib.ace_experts_workspace_size.argtypes = [_P(ace_layer), ctypes.c_int]
_lib.ace_experts_workspace_size.restype = ctypes.c_size_t
_lib.ace_moe_experts.argtypes = [_P(ace_layer), _vp, ctypes.c_int, _vp, _vp, _vp, _vp,
                                 ctypes.c_size_t, _vp]
_lib.ace_moe_experts.restype = ctypes.c_int
_lib.ace_moe_combine.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp,
                                 ctypes.c_int, _vp, _vp, ctypes.c_size_t, _vp]
_lib.ace_moe_combine.restype = ctypes.c_int
_lib.ace_tables_save.argtypes = [ctypes.c_char_p, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp]
_lib.ace_tables_save.restype = ctypes.c_int
_lib.ace_tables_info.argtypes = [ctypes.c_char_p, _P(ctypes.c_int), _P(ctypes.c_int),
                                 _P(ctypes.c_int)]
_lib.ace_tables_info.restype = ctypes.c_int
_lib.ace_tables_load.argtypes = [ctypes.c_char_p, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp]
_lib.ace_tables_load.restype = ctypes.c_int
_lib.ace_moe_decode_noalloc.argtypes = [_P(ace_layer), _vp, ctypes.c_int, _P(ace_fwd_opts), _vp,
                                        _vp]
_lib.ace_moe_decode_noalloc.restype = ctypes.c_int
_lib.ace_tables_workspace_size.argtypes = [_P(ace_layer)]
_lib.ace_tables_workspace_size.restype = ctypes.c_size_t
_lib.ace_build_tables.argtypes = [_P(ace_layer), ctypes.c_int, _P(ace_table_opts), _vp, _vp, _vp,
                                  _vp, _vp, ctypes.c_size_t, _vp]
_lib.ace_build_tables.restype = ctypes.c_int
_lib.ace_stack_workspace_size.argtypes = [_P(ace_layer), ctypes.c_int, ctypes.c_int]
_lib.ace_stack_workspace_size.restype = ctypes.c_size_t
_lib.ace_moe_stack_forward.argtypes = [_P(ace_layer), ctypes.c_int, _vp, ctypes.c_int,
                                       _P(ace_fwd_opts), _vp, _vp, ctypes.c_size_t, _vp]
_lib.ace_moe_stack_forward.restype = ctypes.c_int
_lib.ace_tau_workspace_size.argtypes = []
_lib.ace_tau_workspace_size.restype = ctypes.c_size_t
_lib.ace_tau_quantile.argtypes = [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp,
                                  ctypes.c_size_t, _vp]
_lib.ace_tau_quantile.restype = ctypes.c_int
_lib.ace_noalloc_read_status.argtypes = [_P(ctypes.c_uint32), _vp]
_lib.ace_noalloc_read_status.restype = ctypes.c_int
_lib.ace_set_peer_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.ace_set_peer_wait_limit_ns.restype = ctypes.c_uint64
_lib.ace_read_status.argtypes = [_vp, ctypes.c_size_t, _P(ctypes.c_uint32), _vp]
_lib.ace_read_status.restype = ctypes.c_int
_lib.ace_status_str.argtypes = [ctypes.c_int]
_lib.ace_status_str.restype = ctypes.c_char_p
_lib.ace_version.restype = ctypes.c_char_p
_lib.ace_last_cuda_error.restype = ctypes.c_char_p


class AceError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        msg = "%s: %s" % (where, ace_status_str(code))
        if code == ACE_ERR_CUDA:
            msg += " (%s)" % _lib.ace_last_cuda_error().decode()
        super().__init__(msg)


def _check(code, where):
    if code != ACE_OK:
        raise AceError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def lib():
    return _lib


def ace_status_str(code):
    return _lib.ace_status_str(int(code)).decode()


def ace_version():
    return _lib.ace_version().decode()


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return ACE_BF16
    if t.dtype == torch.float32:
        return ACE_F32
    raise TypeError("unsupported dtype %s" % t.dtype)


def make_layer(gamma, w_router, w_gate, w_up, w_down, k, amax=None, router_bias=None,
               a_gsp=None, a_rcr=None):
    """Pack device tensors into an ``ace_layer``.  The caller keeps the tensors
    alive while the struct is in use."""
    E, d = w_router.shape
    m = w_gate.shape[1]
    for t in (gamma, w_router, w_gate, w_up, w_down, amax, router_bias, a_gsp, a_rcr):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return ace_layer(d=d, E=E, m=m, k=k, dtype=_dtype_code(w_router), gamma=_ptr(gamma),
                     w_router=_ptr(w_router), router_bias=_ptr(router_bias), w_gate=_ptr(w_gate),
                     w_up=_ptr(w_up), w_down=_ptr(w_down), amax=_ptr(amax), a_gsp=_ptr(a_gsp),
                     a_rcr=_ptr(a_rcr))


def _fusion(f):
    return FUSIONS[f] if isinstance(f, str) else int(f)


def ace_workspace_size(layer, max_tokens):
    return int(_lib.ace_workspace_size(ctypes.byref(layer), int(max_tokens)))


def alloc_workspace(nbytes, device="cuda"):
    """A byte tensor usable as workspace (torch allocations are 256-B aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def ace_moe_forward(layer, u, tau, y, ws, renorm=True, eps_rms=1e-6, dbg=None, stream=None,
                    fusion="max"):
    opts = ace_fwd_opts(tau=float(tau), renorm_topk=int(bool(renorm)), fusion=_fusion(fusion),
                        eps_rms=float(eps_rms))
    code = _lib.ace_moe_forward(ctypes.byref(layer), _ptr(u), int(u.shape[0]), ctypes.byref(opts),
                                _ptr(y), _ptr(ws), ws.numel(),
                                ctypes.byref(dbg) if dbg is not None else None, _stream(stream))
    _check(code, "ace_moe_forward")
    return y


def ace_moe_scores(layer, u, score, ws, topk_idx=None, renorm=True, eps_rms=1e-6, stream=None,
                   fusion="max"):
    opts = ace_fwd_opts(tau=0.0, renorm_topk=int(bool(renorm)), fusion=_fusion(fusion),
                        eps_rms=float(eps_rms))
    code = _lib.ace_moe_scores(ctypes.byref(layer), _ptr(u), int(u.shape[0]), ctypes.byref(opts),
                               _ptr(score), _ptr(topk_idx), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "ace_moe_scores")
    return score


def ace_moe_route(layer, u, tau, x, idx, gate, keep, ws, renorm=True, eps_rms=1e-6, stream=None,
                  fusion="max"):
    """Routing with its decisions (see include/ace.h): x [T][d] the experts'
    input rows, idx / gate [T][k], keep [T][k] uint8."""
    opts = ace_fwd_opts(tau=float(tau), renorm_topk=int(bool(renorm)), fusion=_fusion(fusion),
                        eps_rms=float(eps_rms))
    code = _lib.ace_moe_route(ctypes.byref(layer), _ptr(u), int(u.shape[0]), ctypes.byref(opts),
                              _ptr(x), _ptr(idx), _ptr(gate), _ptr(keep), _ptr(ws), ws.numel(),
                              _stream(stream))
    _check(code, "ace_moe_route")
    return x, idx, gate, keep


def make_expert_layer(w_gate, w_up, w_down):
    """An ``ace_layer`` holding only experts (for ace_moe_experts): E, m, d
    from the weight shapes [E][m][d] and [E][d][m]."""
    for t in (w_gate, w_up, w_down):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    E, m, d = w_gate.shape
    return ace_layer(d=d, E=E, m=m, k=1, dtype=_dtype_code(w_gate), gamma=None, w_router=None,
                     router_bias=None, w_gate=_ptr(w_gate), w_up=_ptr(w_up), w_down=_ptr(w_down),
                     amax=None, a_gsp=None, a_rcr=None)


def ace_experts_workspace_size(layer, max_slots):
    return int(_lib.ace_experts_workspace_size(ctypes.byref(layer), int(max_slots)))


def ace_moe_experts(layer, xp, offsets, slot_gate, yslot, ws, stream=None):
    """yslot[s] = slot_gate[s] * f_e(xp[s]) for the slots of expert e,
    offsets[e] <= s < offsets[e + 1] (see include/ace.h); yslot [S][d] in
    xp's dtype."""
    if yslot.dtype != xp.dtype:
        raise ValueError("yslot must have xp's dtype")
    code = _lib.ace_moe_experts(ctypes.byref(layer), _ptr(xp), int(xp.shape[0]), _ptr(offsets),
                                _ptr(slot_gate), _ptr(yslot), _ptr(ws), ws.numel(),
                                _stream(stream))
    _check(code, "ace_moe_experts")
    return yslot


def ace_moe_combine(slot_of, yslot, y, ws, stream=None):
    """y[t] = sum over i of yslot[slot_of[t, i]] for slot_of >= 0, in i order
    (see include/ace.h); slot_of [T][k] int32, yslot [n][d] in y's dtype."""
    if yslot.dtype != y.dtype:
        raise ValueError("yslot must have y's dtype")
    T, k = slot_of.shape
    code = _lib.ace_moe_combine(int(T), int(k), int(y.shape[1]), _dtype_code(y), _ptr(slot_of),
                                _ptr(yslot), int(yslot.shape[0]), _ptr(y), _ptr(ws), ws.numel(),
                                _stream(stream))
    _check(code, "ace_moe_combine")
    return y


def _host_f32(t):
    return t.detach().to("cpu", torch.float32).contiguous()


def ace_tables_save(path, a_gsp, a_rcr, amax, sigma=None):
    """Write ace_build_tables's outputs ([L][E] each, sigma [L][E][3] or None;
    any device) to a tables file (see include/ace.h)."""
    g, r, mx = (_host_f32(t).reshape(-1, a_gsp.shape[-1]) for t in (a_gsp, a_rcr, amax))
    L, E = g.shape
    sg = None if sigma is None else _host_f32(sigma)
    code = _lib.ace_tables_save(os.fsencode(path), L, E, _ptr(g), _ptr(r), _ptr(mx), _ptr(sg))
    _check(code, "ace_tables_save")


def ace_tables_info(path):
    """(n_layers, E, has_sigma) of a tables file."""
    L, E, hs = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    code = _lib.ace_tables_info(os.fsencode(path), ctypes.byref(L), ctypes.byref(E),
                                ctypes.byref(hs))
    _check(code, "ace_tables_info")
    return L.value, E.value, bool(hs.value)


def ace_tables_load(path, device="cpu", with_sigma=False):
    """(a_gsp, a_rcr, amax[, sigma]) from a tables file, fp32 on `device`."""
    L, E, hs = ace_tables_info(path)
    g, r, mx = (torch.empty(L, E, dtype=torch.float32) for _ in range(3))
    sg = torch.empty(L, E, 3, dtype=torch.float32) if with_sigma else None
    code = _lib.ace_tables_load(os.fsencode(path), L, E, _ptr(g), _ptr(r), _ptr(mx), _ptr(sg))
    _check(code, "ace_tables_load")
    out = tuple(t.to(device) for t in (g, r, mx))
    return out + ((sg.to(device),) if with_sigma else ())


def ace_moe_decode_noalloc(layer, u, tau, y, renorm=True, eps_rms=1e-6, stream=None,
                           fusion="max"):
    """Decode forward (1-8 tokens) with the library's fixed scratch array
    instead of a caller workspace; see include/ace.h."""
    opts = ace_fwd_opts(tau=float(tau), renorm_topk=int(bool(renorm)), fusion=_fusion(fusion),
                        eps_rms=float(eps_rms))
    code = _lib.ace_moe_decode_noalloc(ctypes.byref(layer), _ptr(u), int(u.shape[0]),
                                       ctypes.byref(opts), _ptr(y), _stream(stream))
    _check(code, "ace_moe_decode_noalloc")
    return y


def ace_stack_workspace_size(layers, max_tokens):
    arr = (ace_layer * len(layers))(*layers)
    return int(_lib.ace_stack_workspace_size(arr, len(layers), int(max_tokens)))


def ace_moe_stack_forward(layers, u, taus, y, ws, renorm=True, eps_rms=1e-6, stream=None,
                          fusion="max"):
    """len(layers) layers in sequence, each output the next input; taus[l]
    is layer l's threshold.  See include/ace.h."""
    n = len(layers)
    arr = (ace_layer * n)(*layers)
    opts = (ace_fwd_opts * n)(*[ace_fwd_opts(tau=float(t), renorm_topk=int(bool(renorm)),
                                             fusion=_fusion(fusion), eps_rms=float(eps_rms))
                                for t in taus])
    code = _lib.ace_moe_stack_forward(arr, n, _ptr(u), int(u.shape[0]), opts, _ptr(y), _ptr(ws),
                                      ws.numel(), _stream(stream))
    _check(code, "ace_moe_stack_forward")
    return y


def ace_tables_workspace_size(layer):
    return int(_lib.ace_tables_workspace_size(ctypes.byref(layer)))


def ace_build_tables(layers, a_gsp, a_rcr, amax, ws, sigma=None, gsp_norm=ACE_GSP_FRO, eps=1e-6,
                     rho=1.0, power_iters=200, stream=None):
    arr = (ace_layer * len(layers))(*layers)
    opts = ace_table_opts(gsp_norm=gsp_norm, eps=float(eps), rho=float(rho),
                          power_iters=int(power_iters))
    code = _lib.ace_build_tables(arr, len(layers), ctypes.byref(opts), _ptr(a_gsp), _ptr(a_rcr),
                                 _ptr(amax), _ptr(sigma), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "ace_build_tables")


def ace_tau_workspace_size():
    return int(_lib.ace_tau_workspace_size())


def ace_tau_quantile(score, n_skip, tau, ws, stream=None):
    """tau[0] = the (n_skip + 1)-th smallest non-top-1 score of the pool
    score [n_tok][k] (device fp32); see include/ace.h."""
    n_tok, k = score.shape
    code = _lib.ace_tau_quantile(_ptr(score), int(n_tok), int(k), int(n_skip), _ptr(tau),
                                 _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "ace_tau_quantile")
    return tau


def ace_read_status(ws, stream=None):
    """Synchronise the stream; return (status code, flag bits)."""
    flags = ctypes.c_uint32(0)
    code = _lib.ace_read_status(_ptr(ws), ws.numel(), ctypes.byref(flags), _stream(stream))
    return code, int(flags.value)


def ace_noalloc_read_status(stream=None):
    """Synchronise the stream; (status code, flag bits) of the last
    ace_moe_decode_noalloc call on the current device."""
    flags = ctypes.c_uint32(0)
    code = _lib.ace_noalloc_read_status(ctypes.byref(flags), _stream(stream))
    return code, int(flags.value)


def ace_set_peer_wait_limit_ns(ns):
    """Set the limit of cross-CTA waits (0: the 2 s default); returns the
    previous limit."""
    return int(_lib.ace_set_peer_wait_limit_ns(int(ns)))


class DebugOut:
    """Device buffers for the forward's intermediates, and the C struct that
    points at them."""

    def __init__(self, T, k, E, device="cuda"):
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.topk_idx = torch.empty(T, k, **i32)
        self.gate = torch.empty(T, k, **f32)
        self.score = torch.empty(T, k, **f32)
        self.keep = torch.empty(T, k, dtype=torch.uint8, device=device)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.slot_token = torch.empty(max(T * k, 1), **i32)
        self.slot_rank = torch.empty(max(T * k, 1), **i32)
        self.n_kept = torch.empty(1, **i32)
        self.logits = torch.empty(T, E, **f32)
        self.c = ace_debug_out(**{f: _ptr(getattr(self, f)) for f, _ in ace_debug_out._fields_
                                  if not f.startswith("ev_") and f != "trace"})


def event_handle(ev):
    """The cudaEvent_t behind a torch.cuda.Event, as a void* for the C ABI
    (torch creates the CUDA event at its first record, so record it once)."""
    if not ev.cuda_event:
        ev.record()
    return ctypes.c_void_p(ev.cuda_event)


def timing_debug(ev_begin, ev_mid, ev_end):
    """An ace_debug_out that only records the expert-GEMM timing events."""
    return ace_debug_out(ev_experts_begin=event_handle(ev_begin),
                         ev_experts_mid=event_handle(ev_mid),
                         ev_experts_end=event_handle(ev_end))
