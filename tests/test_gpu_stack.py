"""The layer stack (ace_moe_stack_forward): each layer's output is the next
layer's input.  It must equal the same layers run one call at a time (bit
for bit), replay identically from a CUDA graph, and follow the oracle's own
chain of layers (each oracle output rounded to bf16 before the next layer)
on every token whose routing and mask agree at every layer."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import midpoint_tau

pytestmark = pytest.mark.gpu

W = workloads.Workload


def _layers(w, n, device="cuda"):
    from token_dynamic_expert_b200 import ace
    out = []
    for l in range(n):
        L = workloads.make_layer(w, seed=100 + l, device=device)
        e = torch.arange(w.E, device=device, dtype=torch.float32)
        L["a_gsp"] = 0.5 + (e * 7 % 11) / 10.0
        L["a_rcr"] = 0.6 + (e * 5 % 13) / 12.0
        L["amax"] = torch.maximum(L["a_gsp"], L["a_rcr"])
        L["c"] = ace.make_layer(L["gamma"], L["wr"], L["wg"], L["wu"], L["wd"], w.k,
                                amax=L["amax"], router_bias=L["bias"])
        out.append(L)
    return out


def _chain_by_calls(layers, u, taus, dbgs=None):
    from token_dynamic_expert_b200 import ace
    ws = ace.alloc_workspace(max(ace.ace_workspace_size(L["c"], u.shape[0]) for L in layers))
    x = u
    for l, L in enumerate(layers):
        y = torch.empty_like(u)
        ace.ace_moe_forward(L["c"], x, taus[l], y, ws, dbg=dbgs[l].c if dbgs else None)
        assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
        x = y
    return x


@pytest.mark.parametrize("w,n", [
    (workloads.WORKLOADS["decode_bs8"], 4),
    (workloads.WORKLOADS["decode_bs1"], 3),
    (W("stack_prefill", T=300, d=256, E=16, m=256, k=4, dtype="bf16", bias=True, skip=0.5,
       skip_of="slots"), 3)])
def test_stack_equals_layer_by_layer_and_graph_replay(w, n):
    from token_dynamic_expert_b200 import ace
    layers = _layers(w, n)
    u = workloads.make_tokens(w, token_seed=321, device="cuda")
    taus = [0.05 + 0.02 * l for l in range(n)]
    ref = _chain_by_calls(layers, u, taus)
    cs = [L["c"] for L in layers]
    ws = ace.alloc_workspace(ace.ace_stack_workspace_size(cs, w.T))
    ws.fill_(0xFF)
    y = torch.full_like(u, float("nan"))
    ace.ace_moe_stack_forward(cs, u, taus, y, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert torch.equal(y, ref)
    # captured once, replayed twice
    s = torch.cuda.Stream()
    y2 = torch.full_like(u, float("nan"))
    with torch.cuda.stream(s):
        ace.ace_moe_stack_forward(cs, u, taus, y2, ws, stream=s)  # warm-up outside capture
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ace.ace_moe_stack_forward(cs, u, taus, y2, ws, stream=s)
        y2.fill_(float("nan"))
        g.replay()
        g.replay()
    s.synchronize()
    assert torch.equal(y2, ref)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)


def test_stack_follows_the_oracle_chain():
    from token_dynamic_expert_b200 import ace
    w = W("stack_oracle", T=40, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    n = 3
    layers = _layers(w, n)
    u = workloads.make_tokens(w, token_seed=55, device="cpu")
    cpu = [{k: (v.cpu() if torch.is_tensor(v) else v) for k, v in L.items() if k != "c"}
           for L in layers]
    # the oracle's chain: thresholds from its own scores, outputs rounded to bf16
    taus, refs, x = [], [], u
    for l in range(n):
        Ag, Ar = cpu[l]["a_gsp"].numpy(), cpu[l]["a_rcr"].numpy()
        r0 = oracle.moe_forward(cpu[l], x, 0.0, Ag, Ar, outputs=False)
        tau = midpoint_tau(r0["c"], oracle.n_skip_for(w.T, w.k, w.skip))
        r = oracle.moe_forward(cpu[l], x, tau, Ag, Ar)
        taus.append(tau)
        refs.append(r)
        x = torch.from_numpy(r["y"]).to(torch.bfloat16)
    # the GPU: the stack, and the same layers call by call for their masks
    dbgs = [ace.DebugOut(w.T, w.k, w.E) for _ in range(n)]
    ud = u.cuda()
    chained = _chain_by_calls(layers, ud, taus, dbgs)
    cs = [L["c"] for L in layers]
    ws = ace.alloc_workspace(ace.ace_stack_workspace_size(cs, w.T))
    y = torch.empty_like(ud)
    ace.ace_moe_stack_forward(cs, ud, taus, y, ws)
    torch.cuda.synchronize()
    assert torch.equal(y, chained)
    agree = np.ones(w.T, dtype=bool)
    for l in range(n):
        agree &= np.all(dbgs[l].topk_idx.cpu().numpy() == refs[l]["idx"], axis=1)
        agree &= np.all(dbgs[l].keep.cpu().numpy() == refs[l]["keep"], axis=1)
    assert agree.sum() >= 0.8 * w.T, agree.sum()
    yg = y.float().cpu().numpy()[agree]
    yr = refs[-1]["y"][agree]
    rel = np.abs(yg - yr).max(axis=1) / np.maximum(np.abs(yr).max(axis=1), 1e-30)
    print("stack vs oracle chain: tokens", int(agree.sum()), "max rel", rel.max())
    assert rel.max() <= 3e-2
