"""Host logic of bench.py's N-GPU replica mode on CPU: two gloo ranks agree on
the slowest rank's time and on the whole-job throughput (no GPU needed)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, ws, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    times = {0: 120.0, 1: 150.0}        # ms of timed region per rank
    value, slowest = bench.replica_throughput(ws, 10, 1024, times[rank])
    q.put((rank, value, slowest))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, value, slowest in out:
        assert slowest == 150.0
        assert value == pytest.approx(2 * 10 * 1024 / 0.150)


def test_single_rank_needs_no_process_group():
    import bench
    value, slowest = bench.replica_throughput(1, 4, 8, 2.0)
    assert slowest == 2.0 and value == pytest.approx(4 * 8 / 0.002)


def test_profiled_traffic_follows_workload_rate_and_source():
    """The measured DRAM traffic goes only on the line of the workload, kernel
    and skip rate it was captured on, and only while the kernel's source is
    the captured revision."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    for (wl, kern, rate), (path, sha, nbytes) in bench.PROFILED_TRAFFIC.items():
        assert nbytes > 0
        got = bench.profiled_traffic(wl, kern, rate)
        assert got in (nbytes, None)  # None once the source has changed
        assert bench.profiled_traffic(wl, kern, rate + 0.25) is None
        other = "gateup" if kern == "fused" else "fused"
        assert bench.profiled_traffic(wl, other, rate) is None
    assert bench.profiled_traffic("decode_bs1", "fused", 0.6) is None
