"""The expert-parallel entry points on the GPU: ace_moe_route, ace_moe_experts,
ace_moe_combine, and token_dynamic_expert_b200.ep over a one-rank NCCL group.

This run has one GPU, so the group has one rank.  The exchange code then moves
every kept slot to itself.  The multi-rank exchange is covered on the CPU by
test_ep_dispatch.py.

- Routing through ace_moe_route must give the prefill forward's decisions bit
  for bit.  It uses the prefill routing kernels at every token count; at 1-8
  tokens the forward takes the decode kernel, whose router sums differ in
  order, so there the outputs are compared within the parity bound.
- The EP layer (route, dispatch, ace_moe_experts, return, ace_moe_combine) must
  give ace_moe_forward's output: bit for bit when both take the same expert
  kernel, else within the bf16 parity bound.
- The new entry points must reject bad indices with a status flag, not a fault.
"""
import datetime
import socket

import numpy as np
import pytest
import torch

import workloads
from parity_util import gpu_layer, setup_case

pytestmark = pytest.mark.gpu

W = workloads.Workload


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def group():
    import torch.distributed as dist
    from token_dynamic_expert_b200 import build
    build.build()
    dist.init_process_group("nccl", rank=0, world_size=1,
                            init_method="tcp://127.0.0.1:%d" % _free_port(),
                            timeout=datetime.timedelta(seconds=60))
    yield dist.group.WORLD
    dist.destroy_process_group()


def _rel(y, ref):
    y, ref = y.float().cpu().numpy(), ref.float().cpu().numpy()
    num = np.abs(y - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max())


@pytest.mark.parametrize("T,exact", [(64, True), (4, False), (640, False)])
def test_ep_layer_matches_forward(group, T, exact):
    from token_dynamic_expert_b200 import ace, ep
    w = W("ep", T=T, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, _, _, amax, tau, _ = setup_case(w, tables="spread")
    g, c = gpu_layer(layer, amax)
    ud = u.cuda()
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, T))
    # the forward, with its decisions
    dbg = ace.DebugOut(T, w.k, w.E, "cuda")
    y_ref = torch.full_like(ud, float("nan"))
    ace.ace_moe_forward(c, ud, tau, y_ref, ws, dbg=dbg.c)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    # routing alone: the same bits
    x = torch.empty_like(ud)
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    keep = torch.empty(T, w.k, dtype=torch.uint8, device="cuda")
    ace.ace_moe_route(c, ud, tau, x, idx, gate, keep, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    if T > 8:  # the forward's prefill route: the same routing kernels
        assert torch.equal(idx, dbg.topk_idx)
        assert torch.equal(gate, dbg.gate)
        assert torch.equal(keep, dbg.keep)
    # the experts' input rows are bf16(RMSNorm(u) * gamma)
    xr = (u.double() / torch.sqrt((u.double() ** 2).mean(1, keepdim=True) + 1e-6) *
          layer["gamma"].double())
    assert _rel(x, xr) <= 1e-2
    # the EP layer on one rank
    el = ace.make_expert_layer(g["wg"], g["wu"], g["wd"])
    ws_e = ace.alloc_workspace(ace.ace_experts_workspace_size(el, T * w.k))
    y = ep.ep_layer_forward(c, el, ud, tau, ws, ws_e, group=group)
    torch.cuda.synchronize()
    assert ace.ace_read_status(ws_e) == (ace.ACE_OK, 0)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert torch.isfinite(y.float()).all()
    if exact:
        assert torch.equal(y, y_ref)
    else:
        assert _rel(y, y_ref) <= 2e-2


def test_experts_and_combine_flag_bad_indices():
    from token_dynamic_expert_b200 import ace, build
    build.build()
    w = W("ep_bad", T=16, d=256, E=8, m=256, k=2, dtype="bf16", bias=False, skip=0.0,
          skip_of="slots")
    layer = workloads.make_layer(w, seed=4, device="cuda")
    el = ace.make_expert_layer(layer["wg"], layer["wu"], layer["wd"])
    S = 12
    xp = torch.randn(S, w.d, device="cuda").to(torch.bfloat16)
    g = torch.ones(S, device="cuda")
    ws = ace.alloc_workspace(ace.ace_experts_workspace_size(el, S))
    # offsets that do not end at S
    bad = torch.tensor([0, 3, 5, 5, 9, 9, 10, 11, 11], dtype=torch.int32, device="cuda")
    ys = torch.zeros(S, w.d, dtype=torch.bfloat16, device="cuda")
    ace.ace_moe_experts(el, xp, bad, g, ys, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_ERR_DEVICE_FAULT, ace.ACE_FLAG_BAD_INDEX)
    # good offsets: clean, finite
    good = torch.tensor([0, 3, 5, 5, 9, 9, 10, 11, 12], dtype=torch.int32, device="cuda")
    ace.ace_moe_experts(el, xp, good, g, ys, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert torch.isfinite(ys).all()
    # combine: an index past the rows drops out with a flag
    slot_of = torch.tensor([[0, 1], [2, -1], [S + 5, 3]], dtype=torch.int32, device="cuda")
    y = torch.empty(3, w.d, dtype=torch.bfloat16, device="cuda")
    ace.ace_moe_combine(slot_of, ys, y, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_ERR_DEVICE_FAULT, ace.ACE_FLAG_BAD_INDEX)
    assert torch.equal(y[2], ys[3])
    assert torch.equal(y[1], ys[2])
