"""ace_moe_decode_noalloc: the decode forward for callers that cannot
allocate device memory (a host framework that owns every allocation, a
serving loop that must not allocate while running).  Its scratch is a fixed
array compiled into the library, so its results must equal those of
ace_moe_forward with a caller workspace.  Two calls in a row check that the
shared array's leftovers from one call do not leak into the next.

This file is collected last on purpose: a failure here comes after every
other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _rel(y, ref):
    y = y.float().cpu().numpy()
    ref = ref.float().cpu().numpy()
    num = np.abs(y - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max())


@pytest.mark.parametrize("T", [1, 8])
def test_noalloc_decode_matches_workspace_forward(T):
    from token_dynamic_expert_b200 import build
    build.build()
    from token_dynamic_expert_b200 import ace
    w = workloads.WORKLOADS["decode_bs8"].with_(T=T)
    layer = workloads.make_layer(w, seed=21, device="cuda")
    e = torch.arange(w.E, device="cuda", dtype=torch.float32)
    amax = 0.8 + (e * 7 % 11) / 20.0
    L = ace.make_layer(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], w.k,
                       amax=amax)
    tau = 0.12
    ws = ace.alloc_workspace(ace.ace_workspace_size(L, T))
    for call, seed in enumerate((31, 32)):  # two calls in a row, different tokens
        u = workloads.make_tokens(w, T=T, token_seed=seed, device="cuda")
        y_ref = torch.full_like(u, float("nan"))
        ace.ace_moe_forward(L, u, tau, y_ref, ws)
        y = torch.full_like(u, float("nan"))
        ace.ace_moe_decode_noalloc(L, u, tau, y)
        assert ace.ace_noalloc_read_status() == (ace.ACE_OK, 0), call  # the array's status word
        assert torch.isfinite(y.float()).all()
        assert _rel(y, y_ref) <= 2e-2, (call, _rel(y, y_ref))
        assert torch.equal(y, y_ref), call  # same kernel, same inputs: identical bits


def test_noalloc_rejects_what_it_cannot_serve():
    from token_dynamic_expert_b200 import ace
    w = workloads.WORKLOADS["decode_bs8"]
    layer = workloads.make_layer(w.with_(E=16), seed=2, device="cuda")
    L = ace.make_layer(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], w.k)
    u = torch.zeros(9, w.d, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros_like(u)
    opts = ace.ace_fwd_opts(tau=0.1, renorm_topk=1, fusion=0, eps_rms=1e-6)
    f = ace.lib().ace_moe_decode_noalloc
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert f(ctypes.byref(L), ctypes.c_void_p(u.data_ptr()), 9, ctypes.byref(opts),
             ctypes.c_void_p(y.data_ptr()), s) == ace.ACE_ERR_INVALID_ARG  # T > 8
    assert f(ctypes.byref(L), ctypes.c_void_p(u.data_ptr()), 0, ctypes.byref(opts),
             ctypes.c_void_p(y.data_ptr()), s) == ace.ACE_ERR_INVALID_ARG
    assert f(ctypes.byref(L), ctypes.c_void_p(u.data_ptr()), 4, ctypes.byref(opts),
             ctypes.c_void_p(u.data_ptr()), s) == ace.ACE_ERR_INVALID_ARG  # u, y overlap
    # A layer the decode kernel does not serve (hidden size above 2048).  Its
    # buffers are real and of its own shape, so nothing would be read out of
    # bounds even if the call were (wrongly) accepted.
    big = workloads.Workload("big", T=8, d=4096, E=8, m=128, k=2, dtype="bf16", bias=False,
                             skip=0.5, skip_of="slots")
    lb = workloads.make_layer(big, seed=3, device="cuda")
    Lb = ace.make_layer(lb["gamma"], lb["wr"], lb["wg"], lb["wu"], lb["wd"], big.k)
    ub = torch.zeros(8, big.d, dtype=torch.bfloat16, device="cuda")
    yb = torch.zeros_like(ub)
    assert f(ctypes.byref(Lb), ctypes.c_void_p(ub.data_ptr()), 8, ctypes.byref(opts),
             ctypes.c_void_p(yb.data_ptr()), s) == ace.ACE_ERR_UNSUPPORTED
    # the shape rule of ace_moe_forward: bf16 layers need d and m multiples of 128
    odd = workloads.Workload("odd", T=4, d=192, E=16, m=128, k=4, dtype="bf16", bias=False,
                             skip=0.5, skip_of="slots")
    lo = workloads.make_layer(odd, seed=4, device="cuda")
    Lo = ace.make_layer(lo["gamma"], lo["wr"], lo["wg"], lo["wu"], lo["wd"], odd.k)
    uo = torch.zeros(4, odd.d, dtype=torch.bfloat16, device="cuda")
    yo = torch.zeros_like(uo)
    assert f(ctypes.byref(Lo), ctypes.c_void_p(uo.data_ptr()), 4, ctypes.byref(opts),
             ctypes.c_void_p(yo.data_ptr()), s) == ace.ACE_ERR_UNSUPPORTED
    wso = ace.alloc_workspace(1 << 20)
    with pytest.raises(ace.AceError) as ei:
        ace.ace_moe_forward(Lo, uo, 0.1, yo, wso)
    assert ei.value.code == ace.ACE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
