"""The decode kernel's cross-CTA words in the workspace need no clearing.

The decode route of ace_moe_forward launches no clearing kernel: its grid
barriers count in words of the caller's workspace that the last CTA of each
launch leaves zeroed and marked clean for the next launch, and a workspace
without that mark (never used, cleared by another route, or holding anything
else) is handled by a tagged slow path for one launch.  Whatever the
workspace held before, every call must give the same output and a clean
status, and so must calls that alternate with the prefill route (which
clears the same block of words itself).
"""
import pytest
import torch

import workloads
from parity_util import gpu_layer, setup_case

pytestmark = pytest.mark.gpu

W = workloads.Workload


@pytest.fixture(scope="module")
def case():
    from token_dynamic_expert_b200 import build
    build.build()
    from token_dynamic_expert_b200 import ace
    w = W("sync", T=64, d=256, E=16, m=256, k=4, dtype="bf16", bias=False, skip=0.5,
          skip_of="slots")
    layer, u, _, _, amax, tau, _ = setup_case(w, tables="spread")
    g, c = gpu_layer(layer, amax)
    ud = u.cuda()
    ws_bytes = ace.ace_workspace_size(c, w.T)
    ref = {}
    for T in (1, 5, w.T):
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
        y = torch.full_like(ud[:T], float("nan"))
        ace.ace_moe_forward(c, ud[:T], tau, y, ws)
        assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
        ref[T] = y
    # g holds the device weights that c points to: keep it alive with c
    return dict(g=g, c=c, u=ud, tau=tau, ws_bytes=ws_bytes, ref=ref)


def _fill(ws, how):
    if how == "ones":
        ws.fill_(0xFF)
    elif how == "zeros":
        ws.zero_()
    else:  # seeded random bytes
        gen = torch.Generator(device="cpu").manual_seed(7)
        ws.copy_(torch.randint(0, 256, ws.shape, generator=gen, dtype=torch.uint8))


@pytest.mark.parametrize("how", ["zeros", "ones", "random"])
@pytest.mark.parametrize("T", [1, 5])
def test_decode_any_prior_workspace_contents(case, how, T):
    from token_dynamic_expert_b200 import ace
    ws = torch.empty(case["ws_bytes"], dtype=torch.uint8, device="cuda")
    _fill(ws, how)
    for call in range(3):  # the first call takes the slow path, the next ones the fast one
        y = torch.full_like(case["u"][:T], float("nan"))
        ace.ace_moe_forward(case["c"], case["u"][:T], case["tau"], y, ws)
        assert ace.ace_read_status(ws) == (ace.ACE_OK, 0), (how, call)
        assert torch.equal(y, case["ref"][T]), (how, call)


def test_decode_alternating_with_prefill(case):
    """Prefill calls clear the block of words the decode kernel uses; the
    decode calls after them must still synchronise correctly."""
    from token_dynamic_expert_b200 import ace
    ws = torch.empty(case["ws_bytes"], dtype=torch.uint8, device="cuda")
    _fill(ws, "ones")
    T_big = max(case["ref"])
    for T in (1, T_big, 5, 5, T_big, 1, 1):
        y = torch.full_like(case["u"][:T], float("nan"))
        ace.ace_moe_forward(case["c"], case["u"][:T], case["tau"], y, ws)
        assert ace.ace_read_status(ws) == (ace.ACE_OK, 0), T
        assert torch.equal(y, case["ref"][T]), T


def test_decode_graph_replays_stay_clean(case):
    """A captured decode forward replays many times on one workspace: each
    launch leaves the words clean for the next."""
    from token_dynamic_expert_b200 import ace
    ws = torch.empty(case["ws_bytes"], dtype=torch.uint8, device="cuda")
    _fill(ws, "random")
    s = torch.cuda.Stream()
    y = torch.full_like(case["u"][:5], float("nan"))
    with torch.cuda.stream(s):
        ace.ace_moe_forward(case["c"], case["u"][:5], case["tau"], y, ws, stream=s)
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            ace.ace_moe_forward(case["c"], case["u"][:5], case["tau"], y, ws, stream=s)
        for _ in range(50):
            graph.replay()
        s.synchronize()
    del graph
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    assert torch.equal(y, case["ref"][5])
