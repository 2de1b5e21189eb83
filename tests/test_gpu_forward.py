"""GPU parity of ace_moe_forward (through the C ABI) against the fp64 oracle.

Sizes span several tiles and ragged tails; the full-size cases run in the
launch configuration the benchmark times and compare every token's routing
and mask, and a sample of tokens' outputs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, midpoint_tau, run_gpu, setup_case

pytestmark = pytest.mark.gpu

W = workloads.Workload


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_dynamic_expert_b200 import build
    build.build()


def _check(w, tables="oracle", rate=None, T=None, renorm=True, seed=0, y_tol=2e-2,
           out_tokens=None):
    layer, u, A_gsp, A_rcr, amax, tau, n = setup_case(w, seed=seed, T=T, tables=tables, rate=rate,
                                                      renorm=renorm)
    gpu = run_gpu(layer, u, amax, tau, renorm=renorm)
    res = compare(layer, u, gpu, A_gsp, A_rcr, tau, renorm=renorm, y_tol=y_tol,
                  out_tokens=out_tokens)
    print(w.name, res)
    skipped = int((gpu["keep"] == 0).sum())
    if res["band"] == 0 and res["ties"] == 0 and np.isfinite(tau) and tau > 0:
        assert skipped == n  # the threshold realises exactly the requested count
    return res, gpu


# ------------------------------------------------------------ fusion rules
@pytest.mark.parametrize("fusion", ["max", "max_views", "min", "mean", "gsp", "rcr"])
@pytest.mark.parametrize("T", [300, 5])
def test_fusion_rules(fusion, T):
    """The pages' fusion ablation (min, mean) and single views (GSP, RCR)
    next to ACE's max, through the prefill path (300 tokens) and the decode
    kernel (5 tokens), with the view tables given separately; spread tables
    so that the views disagree often."""
    w = W("fusion", T=T, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    # "max_views": ACE's rule with no precomputed max table, only the views
    rule = "max" if fusion == "max_views" else fusion
    layer, u, A_gsp, A_rcr, amax, tau, n = setup_case(w, tables="spread", fusion=rule)
    gpu = run_gpu(layer, u, amax if fusion == "max" else None, tau, fusion=rule,
                  views=(A_gsp, A_rcr))
    res = compare(layer, u, gpu, A_gsp, A_rcr, tau, fusion=rule)
    print(fusion, T, res)
    assert res["mask_mismatch"] == 0
    if res["band"] == 0 and res["ties"] == 0:
        assert int((gpu["keep"] == 0).sum()) == n


def test_tiny_fp32_layer():
    """hidden 256, 8 experts of FFN 128, top-2, 64 tokens, fp32; tau skips
    50% of the non-top-1 slots."""
    res, gpu = _check(workloads.WORKLOADS["tiny_fp32"], y_tol=1e-4)
    assert res["compared_tokens"] == 64
    assert int((gpu["keep"][:, 1] == 0).sum()) == 32


@pytest.mark.parametrize("w", [
    W("multi_tile", T=300, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
      skip_of="slots"),
    W("wide", T=200, d=512, E=8, m=384, k=2, dtype="bf16", bias=False, skip=0.3, skip_of="slots"),
])
def test_bf16_small_layers_oracle_tables(w):
    res, _ = _check(w)
    assert res["compared_tokens"] >= w.T - 2


@pytest.mark.parametrize("E,T,d", [(320, 200, 512), (256, 160, 512), (96, 2000, 256)])
def test_bf16_many_experts_topk_forms(E, T, d):
    """The top-k kernel's forms: 257-512 experts (16 logits a lane), 256 experts
    at a short token count (8 router splits: all of a lane's split loads in
    flight at once) and 96 experts at a long one (4 splits: the 64-register
    form), each against the oracle's routing, mask, slot lists and outputs."""
    w = W("many_experts", T=T, d=d, E=E, m=128, k=8, dtype="bf16", bias=True, skip=0.5,
          skip_of="slots")
    res, gpu = _check(w, tables="spread")
    assert res["compared_tokens"] >= T - 4


def test_bf16_expert_with_several_slot_tiles():
    """8 experts, top-2, 1100 tokens: ~275 slots per expert, so every expert
    spans two tiles of ~138 slots."""
    w = W("heavy", T=1100, d=256, E=8, m=128, k=2, dtype="bf16", bias=False, skip=0.1,
          skip_of="slots")
    res, gpu = _check(w, tables="spread")
    counts = np.diff(gpu["expert_offsets"])
    assert (counts > 256).any()


def test_bf16_router_bias_skewed_load():
    w = W("skewed", T=512, d=384, E=32, m=128, k=4, dtype="bf16", bias=True, skip=0.5,
          skip_of="slots")
    res, gpu = _check(w, tables="spread")
    counts = np.diff(gpu["expert_offsets"])
    assert counts.max() > 3 * max(1, counts.mean())  # the bias does skew the load


@pytest.mark.parametrize("rate", [0.0, 0.75, 0.875])
def test_skip_extremes(rate):
    """0%: every slot kept (dense top-k MoE); 87.5% with k = 8: only top-1."""
    w = W("extremes", T=96, d=256, E=16, m=128, k=8, dtype="bf16", bias=False, skip=rate,
          skip_of="slots")
    res, gpu = _check(w, rate=rate)
    if rate == 0.0:
        assert (gpu["keep"] == 1).all()
    if rate == 0.875:
        assert (gpu["keep"][:, 1:] == 0).all()


def test_no_skip_matches_dense_topk_oracle():
    w = W("dense", T=64, d=256, E=8, m=128, k=3, dtype="bf16", bias=False, skip=0.0,
          skip_of="slots")
    layer, u, A_gsp, A_rcr, amax, _, _ = setup_case(w)
    gpu = run_gpu(layer, u, amax, -1.0)
    assert (gpu["keep"] == 1).all()
    ref = oracle.moe_forward(layer, u, -1.0, A_gsp, A_rcr)
    dense = oracle.combine(ref["x"], ref["idx"], ref["gate"], np.ones_like(ref["keep"]),
                           layer["wg"], layer["wu"], layer["wd"])
    rel = np.abs(gpu["y"] - dense).max(1) / np.abs(dense).max(1)
    assert rel.max() < 2e-2


@pytest.mark.parametrize("k", [1, 8])
def test_k_edge_cases(k):
    w = W("k%d" % k, T=70, d=256, E=8, m=128, k=k, dtype="bf16", bias=False, skip=0.4,
          skip_of="slots")
    _check(w, rate=0.4 if k > 1 else 0.0)


def test_raw_softmax_gates():
    w = W("raw", T=128, d=256, E=16, m=128, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    _check(w, renorm=False)


@pytest.mark.parametrize("T", [1, 2, 31, 33])
def test_ragged_token_counts(T):
    w = W("ragged", T=T, d=256, E=16, m=128, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    _check(w, T=T)


def test_zero_tokens_is_a_noop():
    from token_dynamic_expert_b200 import ace
    w = W("empty", T=4, d=256, E=8, m=128, k=2, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer = workloads.make_layer(w)
    amax = np.ones(w.E, dtype=np.float32)
    from parity_util import gpu_layer
    g, c = gpu_layer(layer, amax)
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, 4))
    u = torch.empty(0, w.d, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(0, w.d, dtype=torch.bfloat16, device="cuda")
    ace.ace_moe_forward(c, u, 0.1, y, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)


def test_forward_is_deterministic():
    w = W("det", T=256, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, A_gsp, A_rcr, amax, tau, _ = setup_case(w, tables="spread")
    a = run_gpu(layer, u, amax, tau)
    b = run_gpu(layer, u, amax, tau)
    assert np.array_equal(a["y"], b["y"])
    assert np.array_equal(a["slot_token"], b["slot_token"])


def test_forward_on_a_side_stream():
    w = W("stream", T=100, d=256, E=8, m=128, k=2, dtype="bf16", bias=False, skip=0.3,
          skip_of="slots")
    layer, u, A_gsp, A_rcr, amax, tau, _ = setup_case(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gpu = run_gpu(layer, u, amax, tau, stream=s)
    compare(layer, u, gpu, A_gsp, A_rcr, tau)


# ------------------------------------------------------------ full sizes
def tile_covering_tokens(gpu, n_out, stride=64, seed=0):
    """Tokens whose outputs cover every expert GEMM tile: the tokens of the
    first and last kept slot of each expert and of every 64th slot between,
    topped up with random tokens to n_out.  An expert of several tiles has
    tiles of near-equal size, at least 128 slots each, so each of its tiles
    holds one of these slots."""
    off = gpu["expert_offsets"]
    st = gpu["slot_token"]
    toks = set()
    for e in range(len(off) - 1):
        if off[e + 1] > off[e]:
            toks.update(int(st[a]) for a in range(off[e], off[e + 1], stride))
            toks.add(int(st[off[e + 1] - 1]))
    T = gpu["keep"].shape[0]
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.fromiter(toks, dtype=np.int64))
    extra = max(0, n_out - len(toks))
    toks.update(rng.choice(rest, size=min(extra, rest.size), replace=False).tolist())
    return np.array(sorted(toks))


def _full(w, n_out=None, seed=0):
    """Full-size layer drawn on the GPU (the CPU copy feeds the oracle); RCR
    table from the oracle, a spread GSP table; every token's routing, mask and
    slot lists compared; outputs on every token (n_out None) or on n_out
    tokens that cover every expert GEMM tile."""
    layer = workloads.make_layer(w, seed=seed, device="cuda")
    u = workloads.make_tokens(w, device="cuda")
    layer_cpu = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in layer.items()}
    u_cpu = u.cpu()
    r = oracle.rcr(layer_cpu["gamma"], layer_cpu["wr"], layer_cpu["wg"], layer_cpu["wu"],
                   layer_cpu["wd"])
    A_rcr = r["A"].astype(np.float32)
    e = np.arange(w.E)
    A_gsp = (0.5 + (e * 7 % 11) / 10.0).astype(np.float32)
    ref = oracle.moe_forward(layer_cpu, u_cpu, 0.0, A_gsp, A_rcr, outputs=False)
    n = oracle.n_skip_for(w.T, w.k, w.skip, of=w.skip_of)
    tau = midpoint_tau(ref["c"], n)
    gpu = run_gpu(layer_cpu, u_cpu, np.maximum(A_gsp, A_rcr), tau)
    toks = None if n_out is None else tile_covering_tokens(gpu, n_out)
    res = compare(layer_cpu, u_cpu, gpu, A_gsp, A_rcr, tau, out_tokens=toks)
    print(w.name, res)
    return res, gpu, n, toks


# The tensor-core router sums exact bf16 x bf16 products of a three-term split
# of the fp32 input in 64-wide chunks, adding chunk sums in fp32: its logits
# must be at least as close to the fp64 definition as an fp32 dot product
# (about 1.5e-6 of the largest logit on these shapes).
ROUTER_TC_REL = 5e-7


def test_full_prefill_1024():
    res, gpu, n, _ = _full(workloads.WORKLOADS["prefill_1024"])
    assert res["compared_tokens"] + res["excluded_tokens"] == 1024  # every token's output
    assert res["slots_checked"] == int(gpu["n_kept"][0])
    assert res["mask_mismatch"] == 0
    assert abs(int((gpu["keep"] == 0).sum()) - n) <= res["band"] + res["ties"] * 8
    assert res["logit_err"] <= ROUTER_TC_REL * res["logit_scale"], res


def test_full_prefill_8192_e256_skewed():
    res, gpu, n, toks = _full(workloads.WORKLOADS["prefill_8192_e256"], n_out=1024)
    counts = np.diff(gpu["expert_offsets"])
    assert counts.max() > 256  # skewed: some experts need several slot tiles
    assert toks.size >= 1024
    assert res["compared_tokens"] + res["excluded_tokens"] == toks.size
    assert res["slots_checked"] == int(gpu["n_kept"][0])
    assert res["logit_err"] <= ROUTER_TC_REL * res["logit_scale"], res


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("T", [1, 2, 3, 8])
def test_full_shape_decode(T):
    """T <= 8 runs the cooperative decode kernel: Qwen3-30B-A3B layer shape,
    every token's routing, mask, slot order and output compared."""
    w = workloads.WORKLOADS["decode_bs8"].with_(T=T)
    layer = workloads.make_layer(w, seed=11, device="cuda")
    layer_cpu = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in layer.items()}
    u_cpu = workloads.make_tokens(w, T=T, token_seed=77)
    r = oracle.rcr(layer_cpu["gamma"], layer_cpu["wr"], layer_cpu["wg"], layer_cpu["wu"],
                   layer_cpu["wd"])
    A_rcr = r["A"].astype(np.float32)
    e = np.arange(w.E)
    A_gsp = (0.5 + (e * 7 % 11) / 10.0).astype(np.float32)
    ref = oracle.moe_forward(layer_cpu, u_cpu, 0.0, A_gsp, A_rcr, outputs=False)
    n = oracle.n_skip_for(T, w.k, 0.6)
    tau = midpoint_tau(ref["c"], n)
    gpu = run_gpu(layer_cpu, u_cpu, np.maximum(A_gsp, A_rcr), tau)
    res = compare(layer_cpu, u_cpu, gpu, A_gsp, A_rcr, tau)
    print("decode", T, res)
    assert res["compared_tokens"] == T


@pytest.mark.parametrize("T", [8, 5, 1])
def test_decode_back_to_back_launches(T):
    """Hundreds of decode launches queued without a synchronisation, each
    with its own workspace: every one finishes without a timeout flag and
    gives the same output as a launch on an idle GPU.  (An odd copy ring once
    let one phase-C warp group lap the other on a shared slot; those waits
    timed out under back-to-back launches only.)"""
    from token_dynamic_expert_b200 import ace
    w = workloads.WORKLOADS["decode_bs8"].with_(T=T)
    layer = workloads.make_layer(w, seed=5, device="cuda")
    u = workloads.make_tokens(w, T=T, token_seed=91, device="cuda")
    amax = torch.linspace(0.6, 1.4, w.E, device="cuda")
    c = ace.make_layer(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], w.k,
                       amax=amax, router_bias=layer["bias"])
    nbytes = ace.ace_workspace_size(c, T)
    tau = 0.08
    y0 = torch.empty_like(u)
    ws0 = ace.alloc_workspace(nbytes)
    ace.ace_moe_forward(c, u, tau, y0, ws0)
    assert ace.ace_read_status(ws0) == (ace.ACE_OK, 0)
    n = 300
    wss = [ace.alloc_workspace(nbytes) for _ in range(n)]
    ys = torch.empty(n, T, w.d, dtype=u.dtype, device="cuda")
    for i in range(n):
        ace.ace_moe_forward(c, u, tau, ys[i], wss[i])
    torch.cuda.synchronize()
    bad = [i for i in range(n) if ace.ace_read_status(wss[i]) != (ace.ACE_OK, 0)]
    assert bad == [], bad[:10]
    assert torch.equal(ys, y0.unsqueeze(0).expand_as(ys))


@pytest.mark.parametrize("T,d", [(2, 384), (6, 384), (3, 128), (7, 2048)])
def test_decode_item_forms_and_strides(T, d):
    """Both forms of the decode kernel's gate/up items: row pairs on the CUDA
    cores below 3 tokens, whole stages on the tensor cores from 3.  The hidden
    sizes give one (d = 128), three (384) and sixteen (2048) groups of four
    32-wide MMA blocks per staged row, and phase-D row counts per CTA of one,
    three and fourteen."""
    w = W("dec_forms", T=T, d=d, E=32, m=128, k=8, dtype="bf16", bias=True, skip=0.5,
          skip_of="slots")
    layer, u, A_gsp, A_rcr, amax, tau, _ = setup_case(w, tables="spread")
    gpu = run_gpu(layer, u, amax, tau)
    res = compare(layer, u, gpu, A_gsp, A_rcr, tau)
    assert res["compared_tokens"] >= T - 1  # run_gpu has checked the status word


@pytest.mark.parametrize("tau", [-1.0, float("inf")])
def test_decode_skip_extremes(tau):
    w = W("dec_ext", T=8, d=256, E=32, m=128, k=8, dtype="bf16", bias=True, skip=0.5,
          skip_of="slots")
    layer, u, A_gsp, A_rcr, amax, _, _ = setup_case(w, tables="spread")
    gpu = run_gpu(layer, u, amax, tau)
    res = compare(layer, u, gpu, A_gsp, A_rcr, tau)
    if tau < 0:
        assert (gpu["keep"] == 1).all()
    else:
        assert (gpu["keep"][:, 1:] == 0).all() and (gpu["keep"][:, 0] == 1).all()
    assert res["compared_tokens"] == 8


def test_decode_in_a_cuda_graph():
    """The forward (decode kernel included) captures into a CUDA graph and
    replays to the same result."""
    from token_dynamic_expert_b200 import ace
    w = W("dec_graph", T=4, d=256, E=16, m=128, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, A_gsp, A_rcr, amax, tau, _ = setup_case(w)
    from parity_util import gpu_layer
    g, c = gpu_layer(layer, amax)
    ud = u.cuda()
    y1 = torch.empty_like(ud)
    y2 = torch.empty_like(ud)
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, w.T))
    ace.ace_moe_forward(c, ud, tau, y1, ws)
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        ace.ace_moe_forward(c, ud, tau, y2, ws, stream=s)
    y2.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
