"""Expert GEMM tiles of every size, through ace_moe_experts with the slot count
of each expert chosen, against the oracle's SwiGLU expert in fp64.

The library cuts an expert's kept slots into ceil(n / 256) tiles of
near-equal size (they differ by one slot at most).  The counts put experts on
both sides of each boundary (16-slot MMA steps, the 64-row slot boxes, one and
several tiles) and include experts with no slot.  Every slot's output row is
compared, so a lost remainder or a misplaced tile shows.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

COUNTS = [0, 1, 15, 16, 17, 63, 65, 255, 256, 257, 300, 383, 384, 385, 520, 800, 0, 1000]
Y_TOL = 2e-2  # row-max relative: bf16 inputs, H and outputs, fp32 accumulation


def _run(E, counts, seed):
    from token_dynamic_expert_b200 import ace, build
    build.build()
    w = workloads.Workload("tiles", T=1, d=256, E=E, m=128, k=1, dtype="bf16", bias=False,
                           skip=0.0, skip_of="slots")
    layer = workloads.make_layer(w, seed=seed, device="cuda")
    el = ace.make_expert_layer(layer["wg"], layer["wu"], layer["wd"])
    counts = np.asarray(counts, dtype=np.int64)
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    S = int(off[-1])
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    xp = torch.randn(S, w.d, device="cuda", generator=g).to(torch.bfloat16)
    gate = torch.rand(S, device="cuda", generator=g) + 0.1
    ys = torch.full((S, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = ace.alloc_workspace(ace.ace_experts_workspace_size(el, S))
    ace.ace_moe_experts(el, xp, torch.from_numpy(off).cuda(), gate, ys, ws)
    assert ace.ace_read_status(ws) == (ace.ACE_OK, 0)
    ys, xp, gate = ys.float().cpu().numpy(), xp.float().cpu().numpy(), gate.cpu().numpy()
    wg, wu, wd = (layer[n].float().cpu().numpy() for n in ("wg", "wu", "wd"))
    worst = 0.0
    for e in range(E):
        for s in range(off[e], off[e + 1]):
            ref = gate[s] * oracle.swiglu(xp[s], wg[e], wu[e], wd[e])[1]
            err = np.abs(ys[s] - ref).max() / max(np.abs(ref).max(), 1e-30)
            worst = max(worst, err)
    assert np.isfinite(ys).all()
    return S, worst


def test_two_launch_tiles():
    """18 experts, 5018 slots: S >= 128 E, so the two-launch kernels run."""
    S, worst = _run(len(COUNTS), COUNTS, seed=11)
    assert S >= 128 * len(COUNTS)
    assert worst <= Y_TOL, worst


def test_fused_tiles():
    """The same counts over 64 experts (the rest empty): S < 128 E, so the
    fused kernel runs."""
    counts = COUNTS + [0] * (64 - len(COUNTS))
    S, worst = _run(64, counts, seed=12)
    assert S < 128 * 64
    assert worst <= Y_TOL, worst
