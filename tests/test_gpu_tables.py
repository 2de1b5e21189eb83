"""GPU parity of ace_build_tables against the fp64 oracle.

GSP (Frobenius and spectral), RCR, their max, and the spectral bound
constants, on small layers (every expert compared) and on the full-size
Qwen3-30B-A3B-shaped layer (RCR for every expert; GSP through ratios of
sampled experts' a~, which the layer normalisation leaves invariant).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu
W = workloads.Workload
RTOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from token_dynamic_expert_b200 import build
    build.build()


def _gpu_tables(layers_cpu, k=2, spectral=False, iters=200, sigma=True, rho=1.0, eps=1e-6):
    from token_dynamic_expert_b200 import ace
    keep = []
    structs = []
    for lc in layers_cpu:
        g = {kk: (v.to("cuda").contiguous() if torch.is_tensor(v) else v) for kk, v in lc.items()}
        keep.append(g)
        structs.append(ace.make_layer(g["gamma"], g["wr"], g["wg"], g["wu"], g["wd"], k,
                                      router_bias=g["bias"]))
    L, E = len(layers_cpu), layers_cpu[0]["E"]
    out = {n: torch.full((L, E), float("nan"), device="cuda") for n in ("a_gsp", "a_rcr", "amax")}
    sig = torch.full((L, E, 3), float("nan"), device="cuda") if sigma else None
    ws = ace.alloc_workspace(ace.ace_tables_workspace_size(structs[0]))
    ws.fill_(0xFF)
    ace.ace_build_tables(structs, out["a_gsp"], out["a_rcr"], out["amax"], ws, sigma=sig,
                         gsp_norm=ace.ACE_GSP_SPECTRAL if spectral else ace.ACE_GSP_FRO,
                         eps=eps, rho=rho, power_iters=iters)
    code, flags = ace.ace_read_status(ws)
    assert code == ace.ACE_OK and flags == 0
    res = {n: t.cpu().numpy() for n, t in out.items()}
    if sigma:
        res["sigma"] = sig.cpu().numpy()
    return res


def _rel(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - b) / np.abs(b)))


@pytest.mark.parametrize("w", [
    W("t_bf16", T=1, d=256, E=16, m=128, k=2, dtype="bf16", bias=False, skip=0.5, skip_of="slots"),
    W("t_bf16_wide", T=1, d=512, E=8, m=384, k=2, dtype="bf16", bias=False, skip=0.5,
      skip_of="slots"),
    W("t_e40", T=1, d=256, E=40, m=256, k=2, dtype="bf16", bias=False, skip=0.5, skip_of="slots"),
    workloads.WORKLOADS["tiny_fp32"],
])
def test_tables_match_oracle(w):
    layer = workloads.make_layer(w, seed=5)
    ref = oracle.tables(layer)
    got = _gpu_tables([layer], k=w.k)
    print(w.name, _rel(got["a_gsp"][0], ref["A_gsp"]), _rel(got["a_rcr"][0], ref["A_rcr"]))
    assert _rel(got["a_gsp"][0], ref["A_gsp"]) < RTOL
    assert _rel(got["a_rcr"][0], ref["A_rcr"]) < RTOL
    assert np.array_equal(got["amax"][0], np.maximum(got["a_gsp"][0], got["a_rcr"][0]))
    sig = oracle.sigma_factors(layer["gamma"], layer["wg"], layer["wu"], layer["wd"], iters=200)
    assert _rel(got["sigma"][0], sig) < RTOL


def test_spectral_gsp_matches_oracle_power_iteration():
    w = W("spec", T=1, d=256, E=8, m=128, k=2, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer = workloads.make_layer(w, seed=9)
    ref = oracle.gsp(layer["gamma"], layer["wg"], layer["wu"], layer["wd"], spectral=True,
                     iters=200)
    got = _gpu_tables([layer], spectral=True, iters=200)
    assert _rel(got["a_gsp"][0], ref["A"]) < RTOL


def test_several_layers_in_one_call():
    w = W("multi", T=1, d=256, E=16, m=128, k=2, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layers = [workloads.make_layer(w, seed=s) for s in (1, 2, 3)]
    got = _gpu_tables(layers, sigma=False)
    for l, lc in enumerate(layers):
        ref = oracle.tables(lc)
        assert _rel(got["a_gsp"][l], ref["A_gsp"]) < RTOL
        assert _rel(got["a_rcr"][l], ref["A_rcr"]) < RTOL


def test_rho_and_scaled_down_projection():
    """Scaling one expert's W^down by 2 doubles its a~ in both views (the
    layer normalisation then shifts every entry)."""
    w = W("scale", T=1, d=256, E=8, m=128, k=2, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer = workloads.make_layer(w, seed=4)
    mod = dict(layer)
    mod["wd"] = layer["wd"].clone()
    mod["wd"][3] *= 2
    a = _gpu_tables([layer], sigma=False)
    b = _gpu_tables([mod], sigma=False)
    for n in ("a_gsp", "a_rcr"):
        ra = a[n][0] / a[n][0][0]
        rb = b[n][0] / b[n][0][0]
        assert abs(rb[3] / ra[3] - 2.0) < 2e-4
    ref = oracle.tables(layer, rho=2.0)
    got = _gpu_tables([layer], sigma=False, rho=2.0)
    assert _rel(got["a_rcr"][0], ref["A_rcr"]) < RTOL


def test_full_size_layer_tables():
    w = workloads.WORKLOADS["prefill_1024"]
    layer = workloads.make_layer(w, seed=0, device="cuda")
    cpu = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in layer.items()}
    got = _gpu_tables([cpu], k=w.k)
    r = oracle.rcr(cpu["gamma"], cpu["wr"], cpu["wg"], cpu["wu"], cpu["wd"])
    assert _rel(got["a_rcr"][0], r["A"]) < RTOL
    # GSP: a~ ratios of sampled experts (normalisation-free), and the mean
    sample = [0, 37, 90, 127]
    g = oracle.gsp(cpu["gamma"], cpu["wg"][sample], cpu["wu"][sample], cpu["wd"][sample])
    ratios_ref = g["a_tilde"] / g["a_tilde"][0]
    ratios = got["a_gsp"][0][sample] / got["a_gsp"][0][sample[0]]
    assert _rel(ratios, ratios_ref) < RTOL
    assert abs(float(np.mean(got["a_gsp"][0], dtype=np.float64)) - 1.0) < 1e-5
    sig = oracle.sigma_factors(cpu["gamma"], cpu["wg"][sample], cpu["wu"][sample],
                               cpu["wd"][sample], iters=200)
    assert _rel(got["sigma"][0][sample], sig) < RTOL


def test_tables_file_round_trip_drives_the_same_forward(tmp_path):
    """Tables built on the GPU, written to a tables file and read back, give
    the same bits and the same forward output as the tables in memory."""
    from token_dynamic_expert_b200 import ace
    w = W("t_io", T=64, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    lc = workloads.make_layer(w, seed=11)
    g = {kk: (v.to("cuda").contiguous() if torch.is_tensor(v) else v) for kk, v in lc.items()}
    s = ace.make_layer(g["gamma"], g["wr"], g["wg"], g["wu"], g["wd"], w.k)
    t = {n: torch.empty(1, w.E, device="cuda") for n in ("a_gsp", "a_rcr", "amax")}
    sig = torch.empty(1, w.E, 3, device="cuda")
    tws = ace.alloc_workspace(ace.ace_tables_workspace_size(s))
    ace.ace_build_tables([s], t["a_gsp"], t["a_rcr"], t["amax"], tws, sigma=sig)
    assert ace.ace_read_status(tws) == (ace.ACE_OK, 0)
    p = str(tmp_path / "layer.acetbl")
    ace.ace_tables_save(p, t["a_gsp"], t["a_rcr"], t["amax"], sig)
    a_gsp, a_rcr, amax, sig2 = ace.ace_tables_load(p, device="cuda", with_sigma=True)
    assert torch.equal(amax, t["amax"]) and torch.equal(sig2, sig)
    assert torch.equal(a_gsp, t["a_gsp"]) and torch.equal(a_rcr, t["a_rcr"])
    u = workloads.make_tokens(w, token_seed=12, device="cuda")
    ys = []
    for am in (t["amax"][0].contiguous(), amax[0].contiguous()):
        L = ace.make_layer(g["gamma"], g["wr"], g["wg"], g["wu"], g["wd"], w.k, amax=am)
        ws = ace.alloc_workspace(ace.ace_workspace_size(L, w.T))
        y = torch.empty_like(u)
        ace.ace_moe_forward(L, u, 0.1, y, ws)
        assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
        ys.append(y)
    assert torch.equal(ys[0], ys[1])
