"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare.

Comparison contract
  * top-k indices: bit-exact, except tokens whose oracle logits have a near
    tie (adjacent gap within the k+1 best below a bound set by the observed
    GPU-vs-oracle logit error); such tokens are counted and left out;
  * skip mask: bit-exact, except slots whose oracle score lies within 1e-6
    relative of tau (counted, expected 0);
  * expert offsets and slot lists: always bit-exact against the oracle's
    compaction of the GPU's own top-k indices and mask (and against the
    oracle's whole routing when every token agrees);
  * outputs: max over compared tokens of ||y - y_ref||_inf / ||y_ref||_inf,
    where y_ref is the oracle's fp64 output (its own mask equals the GPU's
    on every compared token).
Thresholds are the oracle's scores' midpoint between the n-th and (n+1)-th
smallest non-top-1 score, so no slot sits exactly on tau.
"""
import math

import numpy as np
import torch

import oracle
import workloads

BAND = 1e-6


def oracle_tables32(layer_cpu):
    """Oracle GSP/RCR tables rounded to fp32 (the tables both sides read)."""
    t = oracle.tables(layer_cpu)
    a_gsp = t["A_gsp"].astype(np.float32)
    a_rcr = t["A_rcr"].astype(np.float32)
    return a_gsp, a_rcr


def midpoint_tau(c, n_skip):
    cand = np.sort(np.asarray(c)[:, 1:].reshape(-1))
    if n_skip <= 0:
        return float(np.float32(-1.0))
    if n_skip >= cand.size:
        return float(np.float32(np.inf))
    return float(np.float32(0.5 * (cand[n_skip - 1] + cand[n_skip])))


def _dev32(a, device):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def gpu_layer(layer_cpu, amax32, device="cuda", views=None):
    """Device copy of a layer and its ace_layer; views = (A_gsp, A_rcr) fp32
    tables for the fusion rules that read them."""
    from token_dynamic_expert_b200 import ace
    g = {k: (v.to(device).contiguous() if torch.is_tensor(v) else v) for k, v in layer_cpu.items()}
    g["amax"] = _dev32(amax32, device)
    g["a_gsp"], g["a_rcr"] = (_dev32(v, device) for v in (views or (None, None)))
    c = ace.make_layer(g["gamma"], g["wr"], g["wg"], g["wu"], g["wd"], layer_cpu["k"],
                       amax=g["amax"], router_bias=g["bias"], a_gsp=g["a_gsp"], a_rcr=g["a_rcr"])
    return g, c


def run_gpu(layer_cpu, u_cpu, amax32, tau32, renorm=True, ws_tokens=None, stream=None,
            fusion="max", views=None):
    from token_dynamic_expert_b200 import ace
    g, c = gpu_layer(layer_cpu, amax32, views=views)
    u = u_cpu.to("cuda").contiguous()
    T = u.shape[0]
    y = torch.full_like(u, float("nan"))
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, ws_tokens or max(T, 1)))
    ws.fill_(0xFF)  # poison: reads of unwritten scratch show up as NaN
    dbg = ace.DebugOut(T, layer_cpu["k"], layer_cpu["E"])
    ace.ace_moe_forward(c, u, tau32, y, ws, renorm=renorm, dbg=dbg.c, stream=stream,
                        fusion=fusion)
    code, flags = ace.ace_read_status(ws, stream=stream)
    torch.cuda.synchronize()
    assert code == ace.ACE_OK and flags == 0, (ace.ace_status_str(code), flags)
    out = {k: getattr(dbg, k).cpu().numpy() for k in
           ("topk_idx", "gate", "score", "keep", "expert_offsets", "slot_token", "slot_rank",
            "n_kept", "logits")}
    out["y"] = y.float().cpu().numpy()
    out["g"] = g
    out["c"] = c
    return out


def near_tie_tokens(logits, k, tol):
    """Tokens whose k+1 best logits (or the order inside the top k) are
    separated by at most tol somewhere."""
    s = -np.sort(-logits, axis=1)[:, : k + 1]
    gaps = s[:, :-1] - s[:, 1:]
    return np.where((gaps <= tol).any(axis=1))[0]


def compare(layer_cpu, u_cpu, gpu, A_gsp32, A_rcr32, tau32, renorm=True, out_tokens=None,
            y_tol=2e-2, fusion="max"):
    """Compare the GPU forward with the oracle; returns a dict of the counts."""
    T = u_cpu.shape[0]
    k, E = layer_cpu["k"], layer_cpu["E"]
    ref = oracle.moe_forward(layer_cpu, u_cpu, tau32, A_gsp32, A_rcr32, renorm=renorm,
                             outputs=False, fusion=fusion)
    assert ref["disagree"] == 0
    # logits: fp32 GEMM against the fp64 definition
    lerr = np.abs(gpu["logits"] - ref["logits"]).max() if T else 0.0
    scale = max(1.0, np.abs(ref["logits"]).max() if T else 1.0)
    assert lerr <= 2e-5 * scale, lerr
    tol = max(1e-7 * scale, 8 * lerr)
    ties = set(near_tie_tokens(ref["logits"], k, tol).tolist()) if T else set()
    same_idx = np.all(gpu["topk_idx"] == ref["idx"], axis=1)
    bad_idx = [t for t in np.where(~same_idx)[0] if t not in ties]
    assert bad_idx == [], ("top-k differs outside near ties", bad_idx[:10])
    # gates and scores: fp32 against fp64
    ok = same_idx
    if ok.any():
        assert np.allclose(gpu["gate"][ok], ref["gate"][ok], rtol=2e-5, atol=1e-7)
        assert np.allclose(gpu["score"][ok], ref["c"][ok], rtol=2e-5, atol=1e-7)
    # the mask, outside the band around tau
    band = np.abs(ref["c"] - tau32) <= BAND * abs(tau32) if np.isfinite(tau32) else \
        np.zeros_like(ref["c"], dtype=bool)
    mism = (gpu["keep"] != ref["keep"]) & ok[:, None]
    assert not (mism & ~band).any(), ("mask differs outside the band", np.argwhere(mism & ~band)[:10])
    assert (gpu["keep"][:, 0] == 1).all()                 # top-1 always kept
    n_band = int((band & ok[:, None]).sum())
    exact_tokens = ok & ~(mism.any(axis=1))
    res = dict(ties=len(ties), band=n_band, mask_mismatch=int(mism.sum()),
               n_kept=int(gpu["n_kept"][0]), S_ref=ref["S"], logit_err=float(lerr),
               logit_scale=float(scale))
    # compaction of the GPU's own routing: always bit-exact
    own = oracle.compact(gpu["topk_idx"], gpu["keep"], E)
    S_own = own["S"]
    assert int(gpu["n_kept"][0]) == S_own
    assert np.array_equal(gpu["expert_offsets"], own["offsets"])
    assert np.array_equal(gpu["slot_token"][:S_own], own["slot_token"])
    assert np.array_equal(gpu["slot_rank"][:S_own], own["slot_rank"])
    res["slots_checked"] = S_own
    # and identical to the oracle's own routing when every token agrees
    if exact_tokens.all():
        S = ref["S"]
        assert int(gpu["n_kept"][0]) == S
        assert np.array_equal(gpu["expert_offsets"], ref["offsets"])
        assert np.array_equal(gpu["slot_token"][:S], ref["slot_token"])
        assert np.array_equal(gpu["slot_rank"][:S], ref["slot_rank"])
    # outputs on the compared tokens
    toks = np.arange(T) if out_tokens is None else np.asarray(out_tokens)
    n_req = int(toks.size)
    toks = toks[exact_tokens[toks]] if T else toks
    # a requested token is left out only when its top-k flipped on a near tie
    # or a slot of it sits in the band around tau
    res["excluded_tokens"] = n_req - int(toks.size)
    assert res["excluded_tokens"] <= len(ties) + n_band, res
    if toks.size:
        sub = {**layer_cpu}
        yref = oracle.moe_forward(sub, u_cpu[toks], tau32, A_gsp32, A_rcr32, renorm=renorm,
                                  fusion=fusion)["y"]
        y = gpu["y"][toks]
        assert np.isfinite(y).all()
        num = np.abs(y - yref).max(axis=1)
        den = np.maximum(np.abs(yref).max(axis=1), 1e-30)
        rel = float((num / den).max())
        res["y_rel"] = rel
        assert rel <= y_tol, rel
    res["compared_tokens"] = int(toks.size)
    return res


def setup_case(w, seed=0, token_seed=1000, T=None, tables="oracle", rate=None, renorm=True,
               fusion="max"):
    """Layer, tokens, fp32 tables and the midpoint threshold for a workload
    (scores fused by ``fusion``)."""
    layer = workloads.make_layer(w, seed=seed)
    u = workloads.make_tokens(w, T=T, token_seed=token_seed)
    if tables == "oracle":
        A_gsp, A_rcr = oracle_tables32(layer)
    else:  # spread tables: exercise the lookup with a wide range of values
        e = np.arange(w.E)
        A_gsp = (0.5 + (e * 7 % 11) / 10.0).astype(np.float32)
        A_rcr = (0.6 + (e * 5 % 13) / 12.0).astype(np.float32)
    amax = np.maximum(A_gsp, A_rcr)
    rate = w.skip if rate is None else rate
    T_ = u.shape[0]
    ref = oracle.moe_forward(layer, u, 0.0, A_gsp, A_rcr, renorm=renorm, outputs=False,
                             fusion=fusion)
    n = oracle.n_skip_for(T_, w.k, rate, of=w.skip_of)
    tau = midpoint_tau(ref["c"], n)
    return layer, u, A_gsp, A_rcr, amax, tau, n


def realised_skips(keep):
    return int((np.asarray(keep) == 0).sum())


def isfinite(x):
    return math.isfinite(x)
