"""Seeded synthetic workloads for the ACE MoE layer.

This module holds the workload definitions and the seeded input generators
that both the CUDA path and the CPU oracle consume.  It contains none of the
method's arithmetic: only shapes, distributions and the draw order.

Shapes follow the Qwen3-30B-A3B layer (128 routed experts, top-8, hidden 2048,
expert FFN 768) and the 256-expert / FFN-512 layer listed in the architecture
table ("Table 8: Architectures of the evaluated MoE checkpoints") of the ExFold
listing.  The pages measure on real checkpoints and datasets; these random
tensors stand in for them.

Draw order (one generator, seeded per layer; fp32 draws rounded to the storage
dtype with round-to-nearest-even):
    gamma ~ U(0.5, 1.5) [d]
    W_r   ~ N(0, 0.02)  [E, d]
    b     ~ N(0, 1)     [E]          (only when the workload has a router bias)
    W_gate~ N(0, 0.02)  [E, m, d]
    W_up  ~ N(0, 0.02)  [E, m, d]
    W_down~ N(0, 0.02)  [E, d, m]
Tokens are drawn by a second generator seeded with ``token_seed``:
    u     ~ N(0, 1)     [T, d]
gamma and the bias stay fp32; everything else takes the workload dtype.
"""
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens per forward
    d: int            # hidden size
    E: int            # routed experts
    m: int            # expert intermediate size
    k: int            # top-k
    dtype: str        # "bf16" or "f32"
    bias: bool        # router logits carry a per-expert bias
    skip: float       # target skip rate
    skip_of: str      # "slots": of all T*k slots; "nontop1": of the T*(k-1) non-top-1 slots
    seed: int = 0
    layers: int = 1   # independently seeded layers (decode streams 48)
    pool: int = 0     # tokens in the threshold pool (0: the forward's own tokens)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    # fp32 tiny layer: hidden 256, 8 experts of FFN 128, top-2, 64 tokens,
    # tau at the score quantile that skips 50% of the non-top-1 slots
    "tiny_fp32": Workload("tiny_fp32", T=64, d=256, E=8, m=128, k=2, dtype="f32",
                          bias=False, skip=0.5, skip_of="nontop1"),
    # Qwen3-30B-A3B-shaped layer, prefill of 1 x 1024 tokens, 60% skip
    "prefill_1024": Workload("prefill_1024", T=1024, d=2048, E=128, m=768, k=8, dtype="bf16",
                             bias=False, skip=0.6, skip_of="slots"),
    # same layer in decode (1 or 8 tokens per step), 48 independently seeded
    # layers so that weights stream from HBM; tau per layer from a 4096-token pool
    "decode_bs1": Workload("decode_bs1", T=1, d=2048, E=128, m=768, k=8, dtype="bf16",
                           bias=False, skip=0.6, skip_of="slots", layers=48, pool=4096),
    "decode_bs8": Workload("decode_bs8", T=8, d=2048, E=128, m=768, k=8, dtype="bf16",
                           bias=False, skip=0.6, skip_of="slots", layers=48, pool=4096),
    # the same 48 layers chained (each layer's output the next one's input):
    # one step is a token step through the model's MoE layers
    "stack_bs1": Workload("stack_bs1", T=1, d=2048, E=128, m=768, k=8, dtype="bf16",
                          bias=False, skip=0.6, skip_of="slots", layers=48, pool=4096),
    "stack_bs8": Workload("stack_bs8", T=8, d=2048, E=128, m=768, k=8, dtype="bf16",
                          bias=False, skip=0.6, skip_of="slots", layers=48, pool=4096),
    # wider pool: 256 experts of FFN 512, 4 x 2048 tokens, router bias N(0,1)
    # (skewed expert load), 50% skip
    "prefill_8192_e256": Workload("prefill_8192_e256", T=8192, d=2048, E=256, m=512, k=8,
                                  dtype="bf16", bias=True, skip=0.5, skip_of="slots"),
    # skip-rate sweep on the 128 x 768 layer with 4096 prefill tokens
    "sweep_4096": Workload("sweep_4096", T=4096, d=2048, E=128, m=768, k=8, dtype="bf16",
                           bias=False, skip=0.6, skip_of="slots"),
}
SWEEP_RATES = (0.0, 0.25, 0.5, 0.6, 0.75)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_layer(w: Workload, seed: int = None, device="cpu"):
    """Weights of one layer, drawn in the documented order."""
    seed = w.seed if seed is None else seed
    g = _gen(seed, device)
    dt = w.torch_dtype
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    gamma = torch.rand(w.d, **f32) + 0.5
    wr = (torch.randn(w.E, w.d, **f32) * 0.02).to(dt)
    bias = torch.randn(w.E, **f32) if w.bias else None
    wg = (torch.randn(w.E, w.m, w.d, **f32) * 0.02).to(dt)
    wu = (torch.randn(w.E, w.m, w.d, **f32) * 0.02).to(dt)
    wd = (torch.randn(w.E, w.d, w.m, **f32) * 0.02).to(dt)
    return dict(gamma=gamma, wr=wr, bias=bias, wg=wg, wu=wu, wd=wd, k=w.k, d=w.d, E=w.E, m=w.m)


def make_tokens(w: Workload, T: int = None, token_seed: int = 1000, device="cpu"):
    """Layer input rows u ~ N(0, 1) in the workload dtype."""
    T = w.T if T is None else T
    g = _gen(token_seed, device)
    return torch.randn(T, w.d, dtype=torch.float32, device=device, generator=g).to(w.torch_dtype)


def layer_to(layer, device):
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in layer.items()}
