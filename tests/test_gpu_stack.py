"""The layer stack (ace_moe_stack_forward): each layer's output is the next
layer's input.  It must equal the same layers run one call at a time (bit
for bit), replay identically from a CUDA graph, and each layer of it must
match the oracle on that layer's own input."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, midpoint_tau, run_gpu

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


def test_stack_follows_the_oracle_layer_by_layer():
    """Every layer of the chain against the oracle on that layer's own GPU
    input (the bf16 output of the GPU's previous layer): routing, mask and
    slot lists bit-exact outside near ties and the band around tau, outputs
    within 2e-2 on every token; then the stack's output equals that chain of
    calls bit for bit."""
    from token_dynamic_expert_b200 import ace
    w = W("stack_oracle", T=40, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    n = 3
    layers = _layers(w, n)
    u = workloads.make_tokens(w, token_seed=55, device="cpu")
    cpu = [{k: (v.cpu() if torch.is_tensor(v) else v) for k, v in L.items() if k != "c"}
           for L in layers]
    taus, x = [], u
    for l in range(n):
        Ag, Ar = cpu[l]["a_gsp"].numpy(), cpu[l]["a_rcr"].numpy()
        r0 = oracle.moe_forward(cpu[l], x, 0.0, Ag, Ar, outputs=False)
        tau = midpoint_tau(r0["c"], oracle.n_skip_for(w.T, w.k, w.skip))
        gpu = run_gpu(cpu[l], x, np.maximum(Ag, Ar), tau)
        res = compare(cpu[l], x, gpu, Ag, Ar, tau)
        print("layer", l, res)
        assert res["mask_mismatch"] == 0
        assert res["compared_tokens"] + res["excluded_tokens"] == w.T
        taus.append(tau)
        x = torch.from_numpy(gpu["y"]).to(torch.bfloat16)  # bf16 values, exactly
    cs = [L["c"] for L in layers]
    ws = ace.alloc_workspace(ace.ace_stack_workspace_size(cs, w.T))
    ud = u.cuda()
    y = torch.empty_like(ud)
    ace.ace_moe_stack_forward(cs, ud, taus, y, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert torch.equal(y.cpu(), x)
