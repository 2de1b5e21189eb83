"""Expert-parallel dispatch of kept slots (token_dynamic_expert_b200.ep) on the
CPU ([ACE] "Conclusion", future directions: distributed expert dispatch).

Two or four gloo ranks each hold a share of the tokens and of the experts.
Every rank routes its own tokens and sends its kept slots to the experts'
owners.  The owners run their experts, and the outputs come back for the
combine.  The oracle stands in for the experts and for the combine (the
library's kernels do that on the GPU).

The exchange code is the product's own; only the arithmetic is injected.  The
combined outputs must equal the single-process oracle forward bit for bit: both
evaluate g * f_e(x) per kept slot in fp64 and add them in rank order, so any
slot sent to the wrong expert, returned to the wrong token or added out of order
shows.  Skipped slots must not travel: every rank checks that it received
exactly the kept slots of its experts.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case(E=8, T=64, skip_rate=0.5, concentrate=False):
    """Weights, tokens and the full-batch oracle routing, mask and forward."""
    w = workloads.WORKLOADS["tiny_fp32"].with_(E=E, T=T)
    layer = workloads.make_layer(w, seed=3)
    u = workloads.make_tokens(w, token_seed=5)
    _, x = oracle.rmsnorm(u, layer["gamma"])
    _, idx, gate = oracle.router(x, layer["wr"], layer["bias"], w.k)
    if concentrate:  # every slot on the experts of rank 0 (the other ranks receive nothing)
        idx = (np.arange(T * w.k).reshape(T, w.k) % (E // 2)).astype(np.int32)
    e = np.arange(E)
    A = (0.5 + (e * 7 % 11) / 10.0).astype(np.float64)
    c = gate * A[idx]
    tau = oracle.tau_quantile(c, oracle.n_skip_for(T, w.k, skip_rate))
    keep = oracle.mask(idx, gate, A, A, tau)["keep"]
    y = oracle.combine(x, idx, gate, keep, layer["wg"], layer["wu"], layer["wd"])
    wts = {n: layer[n].numpy() for n in ("wg", "wu", "wd")}
    return dict(x=x, idx=idx, gate=gate, keep=keep, y=y, E=E, k=w.k, **wts)


def _rank(rank, world, port, case, q):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as ora
        from token_dynamic_expert_b200 import ep
        T = case["x"].shape[0]
        Tl = T // world
        sl = slice(rank * Tl, (rank + 1) * Tl)
        E, k = case["E"], case["k"]
        per = E // world
        e0 = rank * per
        seen = {}

        def experts_fn(xp, offsets, g):
            off = offsets.numpy()
            seen["n"] = int(off[-1])
            out = np.empty(xp.shape)
            for j in range(per):
                e = e0 + j
                for s in range(off[j], off[j + 1]):
                    f = ora.swiglu(xp[s].numpy(), case["wg"][e], case["wu"][e], case["wd"][e])[1]
                    out[s] = g[s].item() * f
            return torch.from_numpy(out)

        def combine_fn(slot_of, rows):
            so, r = slot_of.numpy(), rows.numpy()
            y = np.zeros((so.shape[0], r.shape[1]))
            for t in range(so.shape[0]):
                for i in range(so.shape[1]):  # rank order
                    if so[t, i] >= 0:
                        y[t] += r[so[t, i]]
            return torch.from_numpy(y)

        y = ep.ep_moe_forward(torch.from_numpy(case["x"][sl]), torch.from_numpy(case["idx"][sl]),
                              torch.from_numpy(case["gate"][sl]), torch.from_numpy(case["keep"][sl]),
                              E, experts_fn, combine_fn)
        q.put((rank, y.numpy(), seen.get("n", 0)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(case, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


@pytest.mark.parametrize("world,E,concentrate", [(2, 8, False), (4, 8, False), (2, 8, True)])
def test_ep_dispatch_equals_single_process_oracle(world, E, concentrate):
    case = _case(E=E, concentrate=concentrate)
    out = _run(case, world)
    y = np.concatenate([o[1] for o in out])
    assert np.array_equal(y, case["y"])
    # each owner ran exactly the kept slots of its experts, no skipped slot travelled
    per = E // world
    kept_e = case["idx"][case["keep"] != 0]
    for rank, _, n in out:
        assert n == int(((kept_e >= rank * per) & (kept_e < (rank + 1) * per)).sum())
    if concentrate:
        assert out[1][2] == 0  # rank 1 owns experts no slot chose


def test_dispatch_plan_order_and_counts():
    from token_dynamic_expert_b200 import ep
    idx = torch.tensor([[5, 1], [0, 7], [1, 4]], dtype=torch.int32)
    keep = torch.tensor([[1, 1], [1, 0], [1, 1]], dtype=torch.uint8)
    slot, e, counts = ep.dispatch_plan(idx, keep, E=8, world=2)
    # kept slots (t*k+i -> expert): 0->5, 1->1, 2->0, 4->1, 5->4; rank 0 owns 0-3
    assert slot.tolist() == [2, 1, 4, 5, 0]
    assert e.tolist() == [0, 1, 1, 4, 5]
    assert counts.tolist() == [3, 2]
