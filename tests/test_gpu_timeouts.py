"""Bounded waits that run out are reported, and leave the GPU usable.

With the limit of the cross-CTA waits set to 1 ns (ace_set_peer_wait_limit_ns),
a CTA that waits on another one gives up at once: the down items of the fused
prefill expert kernel (waiting for their tile's h rows) and the decode
kernel's grid barriers.  Nothing is left waiting: the kernel lets its copies
land, frees its tensor memory and returns with ACE_FLAG_TIMEOUT in the status
word.  The call's status must say ACE_ERR_TIMEOUT, and the next call with the
default limit, on the same workspace, must give the same output as a call
before the timeout.
"""
import numpy as np
import pytest
import torch

import workloads
from parity_util import gpu_layer, setup_case

pytestmark = pytest.mark.gpu

W = workloads.Workload


@pytest.fixture(autouse=True)
def _default_limit():
    from token_dynamic_expert_b200 import build
    build.build()
    from token_dynamic_expert_b200 import ace
    ace.ace_set_peer_wait_limit_ns(0)
    yield
    ace.ace_set_peer_wait_limit_ns(0)


def _timed_out(call, read_status, attempts=3):
    """Run `call` with the 1 ns limit until one reports ACE_ERR_TIMEOUT (a
    wait that happens to find its peers ready needs no limit)."""
    from token_dynamic_expert_b200 import ace
    prev = ace.ace_set_peer_wait_limit_ns(1)
    try:
        for _ in range(attempts):
            call()
            code, flags = read_status()
            assert flags & ~ace.ACE_FLAG_TIMEOUT == 0, flags
            if code == ace.ACE_ERR_TIMEOUT:
                assert flags == ace.ACE_FLAG_TIMEOUT
                return True
            assert code == ace.ACE_OK
        return False
    finally:
        ace.ace_set_peer_wait_limit_ns(prev)


# 96 tokens: the fused expert kernel (T k < 128 E; 64 gate/up and 32 down
# items); 4 tokens: the decode kernel
@pytest.mark.parametrize("T", [96, 4])
def test_peer_wait_timeout_is_reported_and_recovered(T):
    from token_dynamic_expert_b200 import ace
    w = W("timeout", T=T, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, _, _, amax, tau, _ = setup_case(w, tables="spread")
    g, c = gpu_layer(layer, amax)
    ud = u.cuda()
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, T))
    y_ref = torch.full_like(ud, float("nan"))
    ace.ace_moe_forward(c, ud, tau, y_ref, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert ace.ace_set_peer_wait_limit_ns(0) == 2_000_000_000  # the default

    y = torch.empty_like(ud)
    assert _timed_out(lambda: ace.ace_moe_forward(c, ud, tau, y, ws),
                      lambda: ace.ace_read_status(ws))
    # default limit again: the same workspace, the same result as before
    for _ in range(2):
        y2 = torch.full_like(ud, float("nan"))
        ace.ace_moe_forward(c, ud, tau, y2, ws)
        assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
        assert torch.equal(y2, y_ref)


def test_noalloc_timeout_is_visible_and_recovered():
    """The no-allocation decode entry point's status word (in its static
    array) shows the timeout; the next call is clean and equals the
    workspace forward."""
    from token_dynamic_expert_b200 import ace
    w = W("timeout_na", T=4, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, _, _, amax, tau, _ = setup_case(w, tables="spread")
    g, c = gpu_layer(layer, amax)
    ud = u.cuda()
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, w.T))
    y_ref = torch.empty_like(ud)
    ace.ace_moe_forward(c, ud, tau, y_ref, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    y = torch.empty_like(ud)
    assert _timed_out(lambda: ace.ace_moe_decode_noalloc(c, ud, tau, y),
                      ace.ace_noalloc_read_status)
    y2 = torch.full_like(ud, float("nan"))
    ace.ace_moe_decode_noalloc(c, ud, tau, y2)
    assert ace.ace_noalloc_read_status() == (ace.ACE_OK, 0)
    assert torch.equal(y2, y_ref)


def test_timeout_then_graph_replay_is_clean():
    """A limit set at capture time stays in the graph; after a timed-out
    call, a graph captured with the default limit replays cleanly."""
    from token_dynamic_expert_b200 import ace
    w = W("timeout_graph", T=4, d=256, E=16, m=128, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, _, _, amax, tau, _ = setup_case(w, tables="spread")
    g, c = gpu_layer(layer, amax)
    ud = u.cuda()
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, w.T))
    y_ref = torch.empty_like(ud)
    ace.ace_moe_forward(c, ud, tau, y_ref, ws)
    y = torch.empty_like(ud)
    assert _timed_out(lambda: ace.ace_moe_forward(c, ud, tau, y, ws),
                      lambda: ace.ace_read_status(ws))
    s = torch.cuda.Stream()
    y2 = torch.full_like(ud, float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        ace.ace_moe_forward(c, ud, tau, y2, ws, stream=s)
    graph.replay()
    torch.cuda.synchronize()
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert torch.equal(y2, y_ref)
    assert np.isfinite(y2.float().cpu().numpy()).all()
