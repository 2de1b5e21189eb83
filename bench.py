#!/usr/bin/env python
"""Benchmark of the ACE MoE layer forward on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: the Qwen3-30B-A3B-shaped layer (hidden 2048, 128 experts of
FFN 768, top-8, renormalised gates), prefill of 1 x 1024 tokens, 60% of the
T*k slots skipped.  A "step" is one whole forward (RMSNorm, router, top-k,
skip mask, compaction, gate/up GEMM + SiLU, down GEMM x gate, combine) over
the batch.  Inputs are resident in HBM; the weights (1.2 GB) exceed L2, and
L2 is also flushed (a 256 MiB write) before every timed step, outside the
timed interval.  Each step is timed with CUDA events on the launching stream.

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica (the layer forward has no exchange step); the time is the
maximum over ranks and the value counts the tokens of all ranks.
``--impl reference`` times the fp64 CPU oracle on the host cores instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "MoE-layer tokens/s (prefill, decode) at skip rate; % of tensor/HBM roofline"

# DRAM traffic (read + write bytes) per launch of the dominant kernel from one ncu
# capture of that kernel on that workload at that skip rate; reported only while the
# kernel's source is the revision the counters were taken on.
PROFILED_TRAFFIC = {
    ("prefill_1024", "fused", 0.6): ("token_dynamic_expert_b200/csrc/experts_fused_sm100.cu",
                                     "10553744e735", 1227740736),
    # gate/up launch of the 4096-token layer at 0% skip: 1.069221 GB read + 37.43 MB written
    ("sweep_4096", "gateup", 0.0): ("token_dynamic_expert_b200/csrc/experts_sm100.cu",
                                    "7f133c65c8f5", 1106649224),
}


def profiled_traffic(workload, kernel, rate):
    import hashlib
    key = next((k for k in PROFILED_TRAFFIC
                if k[:2] == (workload, kernel) and abs(k[2] - rate) < 1e-9), None)
    if key is None:
        return None
    path, sha, nbytes = PROFILED_TRAFFIC[key]
    with open(os.path.join(ROOT, path), "rb") as f:
        cur = hashlib.sha1(f.read()).hexdigest()[:12]
    return nbytes if cur == sha else None
# rmsnorm (+ the status and bitmap clears), router GEMM, top-k/mask (+ offset scan),
# scatter+gather, the expert GEMMs (one fused launch for small slot tiles, else gate/up
# and down), combine
KERNELS_PER_FORWARD = {True: 6, False: 7}
# per decode layer: the decode kernel alone (its grid-barrier words reset themselves)
KERNELS_PER_DECODE_LAYER = 1


# ----------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=float(j["hbm_gbs"]), bf16_tflops=float(j["bf16_tflops"]),
                    bf16_tflops_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, polled through NVML every
    ~2 ms on a background thread while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.stop = threading.Event()
        self.max_mhz = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:  # NVML unavailable: report unsampled
            self.ok = False
        return self

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self.stop.set()
        if self.ok:
            self.t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml"}


def dist_setup(n):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return ws, rank, local


def max_over_ranks(x, ws):
    """Largest value over the ranks (the slowest replica's time)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(ws, steps, units_per_step, rank_total_ms):
    """Whole-job throughput of N replicas: every rank's units over the
    slowest rank's timed region."""
    slowest = max_over_ranks(rank_total_ms, ws)
    return ws * steps * units_per_step / (slowest / 1e3), slowest


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


# ----------------------------------------------------------- our workload
def step_spread(t_steps, what):
    """Median and max of the timed steps.  A step far above the median means
    a kernel waited out its bounded wait (the status word only holds the last
    call's flags), so the run is rejected rather than averaged."""
    med = float(np.median(t_steps))
    mx = float(np.max(t_steps))
    if mx > 20.0 * med + 1.0:
        raise RuntimeError("%s: a timed step took %.1f ms against a median of %.3f ms"
                           % (what, mx, med))
    return {"median_ms": med, "max_ms": mx}


def tau_on_device(score, n_skip, tws=None):
    """Quantile mapping of the skip count to tau on the GPU (ace_tau_quantile);
    returns a one-element device tensor."""
    from token_dynamic_expert_b200 import ace
    if tws is None:
        tws = ace.alloc_workspace(ace.ace_tau_workspace_size(), score.device)
    tau = torch.empty(1, dtype=torch.float32, device=score.device)
    ace.ace_tau_quantile(score, n_skip, tau, tws)
    return tau


def setup_prefill(w, rate, device):
    from token_dynamic_expert_b200 import ace
    layer = workloads.make_layer(w, seed=w.seed, device=device)
    u = workloads.make_tokens(w, device=device)
    E = w.E
    # ACE tables from the GPU table build
    a_gsp = torch.empty(E, dtype=torch.float32, device=device)
    a_rcr = torch.empty_like(a_gsp)
    amax = torch.empty_like(a_gsp)
    L0 = ace.make_layer(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], w.k,
                        router_bias=layer["bias"])
    tables = "ace_build_tables"
    try:
        tws = ace.alloc_workspace(ace.ace_tables_workspace_size(L0), device)
        ace.ace_build_tables([L0], a_gsp, a_rcr, amax, tws)
        del tws
    except ace.AceError:
        amax.fill_(1.0)
        tables = "unit table (table build unavailable in this build)"
    L = ace.make_layer(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], w.k,
                       amax=amax, router_bias=layer["bias"])
    ws = ace.alloc_workspace(ace.ace_workspace_size(L, w.T), device)
    score = torch.empty(w.T, w.k, dtype=torch.float32, device=device)
    ace.ace_moe_scores(L, u, score, ws)
    torch.cuda.synchronize()
    n_skip = int(np.floor(rate * (w.T * w.k if w.skip_of == "slots" else w.T * (w.k - 1)) + 0.5))
    tau32 = float(tau_on_device(score, n_skip).item())
    y = torch.empty_like(u)
    return dict(layer=layer, u=u, L=L, ws=ws, y=y, tau=tau32, amax=amax, tables=tables,
                n_skip=n_skip)


def slot_stats(st, w):
    """Kept slots and touched experts of one forward (read once, untimed)."""
    from token_dynamic_expert_b200 import ace
    dbg = ace.DebugOut(w.T, w.k, w.E, st["u"].device)
    ace.ace_moe_forward(st["L"], st["u"], st["tau"], st["y"], st["ws"], dbg=dbg.c)
    code, flags = ace.ace_read_status(st["ws"])
    if code != ace.ACE_OK:
        raise RuntimeError("device status %s flags %#x" % (ace.ace_status_str(code), flags))
    off = dbg.expert_offsets.cpu().numpy()
    counts = np.diff(off)
    return dict(S=int(dbg.n_kept.item()), touched=int((counts > 0).sum()),
                skipped=int((dbg.keep == 0).sum().item()), counts=counts)


def pipelined_e2e(st, stream, steps):
    """Milliseconds for `steps` forwards, each with its host-to-device input copy and
    device-to-host output copy, pipelined over two device buffer sets."""
    from token_dynamic_expert_b200 import ace
    dev = st["u"].device
    u_host = st["u"].cpu().pin_memory()
    y_host = torch.empty_like(u_host).pin_memory()
    u_dev = [st["u"], torch.empty_like(st["u"])]
    y_dev = [st["y"], torch.empty_like(st["y"])]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n, t0=None, t1=None):
        h2d.wait_stream(stream)
        if t0 is not None:
            t0.record(h2d)
        for i in range(n):
            b = i % 2
            if i >= 2:
                h2d.wait_event(ev_fwd[b])      # the forward of step i - 2 read u_dev[b]
            with torch.cuda.stream(h2d):
                u_dev[b].copy_(u_host, non_blocking=True)
            ev_in[b].record(h2d)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])   # the output copy of step i - 2 read y_dev[b]
            ace.ace_moe_forward(st["L"], u_dev[b], st["tau"], y_dev[b], st["ws"], stream=stream)
            ev_fwd[b].record(stream)
            d2h.wait_event(ev_fwd[b])
            with torch.cuda.stream(d2h):
                y_host.copy_(y_dev[b], non_blocking=True)
            ev_out[b].record(d2h)
        if t1 is not None:
            t1.record(d2h)
        d2h.synchronize()
        stream.wait_stream(d2h)

    run(2)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, t0, t1)
    return t0.elapsed_time(t1)


def run_ours(args, w, rate, ws_n, rank, local):
    from token_dynamic_expert_b200 import ace
    dev = torch.device("cuda", local)
    st = setup_prefill(w, rate, dev)
    ss = slot_stats(st, w)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def fwd(dbg=None):
        ace.ace_moe_forward(st["L"], st["u"], st["tau"], st["y"], st["ws"], dbg=dbg,
                            stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1)
            fwd()
        code, flags = ace.ace_read_status(st["ws"], stream=stream)
        if code != ace.ACE_OK:
            raise RuntimeError("device status %s flags %#x" % (ace.ace_status_str(code), flags))
        # the whole forward captured once and replayed: one graph launch per step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fwd()
        for _ in range(args.warmup):
            flush.fill_(1)
            graph.replay()
    stream.synchronize()

    # timed: K steps, each bracketed by events on the launching stream
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(ws_n)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.fill_(1)
            evs[i][0].record(stream)
            graph.replay()
            evs[i][1].record(stream)
        stream.synchronize()
    barrier(ws_n)
    t_steps = [a.elapsed_time(b) for a, b in evs]
    spread = step_spread(t_steps, w.name)
    value, total_ms = replica_throughput(ws_n, args.steps, w.T, sum(t_steps))
    ms_step = total_ms / args.steps
    code, flags = ace.ace_read_status(st["ws"], stream=stream)
    if code != ace.ACE_OK:
        raise RuntimeError("device status %s flags %#x" % (ace.ace_status_str(code), flags))

    # per-kernel times of the expert GEMMs, recorded by the library on its stream
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    dbgs = [ace.timing_debug(*e) for e in kev]
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.fill_(1)
            fwd(dbgs[i])
        stream.synchronize()
    t_gu = [e[0].elapsed_time(e[1]) for e in kev]
    t_dn = [e[1].elapsed_time(e[2]) for e in kev]

    # roofline of the dominant kernel (gate/up GEMM + SiLU) and of the down GEMM
    pk = peaks()
    d, m, S, touched = w.d, w.m, ss["S"], ss["touched"]
    gu_bytes = touched * 2 * m * d * 2 + S * d * 2 + S * m * 2
    dn_bytes = touched * d * m * 2 + S * m * 2 + S * d * 2  # bf16 per-slot outputs
    gu_ms = statistics.mean(t_gu)
    dn_ms = statistics.mean(t_dn)
    # small slot tiles: both GEMMs run as one kernel and the library records
    # "mid" after it ("mid" = "end"): the dominant kernel is then the fused one
    fused = dn_ms < 0.02 * gu_ms
    # algorithmic bytes (the method's): the touched experts' weights and the
    # layer's input X and output Y; the design's own intermediates (gathered
    # rows, h, per-slot outputs) are reported beside them
    x_bytes = w.T * d * 2
    if fused:
        kname = "k_experts_fused (gate/up + SiLU and down GEMMs, one launch)"
        k_bytes, k_ms = touched * 3 * m * d * 2 + 2 * x_bytes, gu_ms + dn_ms
        k_bytes_incl = gu_bytes + dn_bytes
    else:
        kname = "k_experts_pair<0> (gate/up GEMM + SiLU, CTA pairs)"
        k_bytes, k_ms = touched * 2 * m * d * 2 + x_bytes, gu_ms
        k_bytes_incl = gu_bytes
    k_gbs = k_bytes / (k_ms / 1e3) / 1e9
    k_gbs_incl = k_bytes_incl / (k_ms / 1e3) / 1e9
    dn_gbs = dn_bytes / (dn_ms / 1e3) / 1e9 if not fused else None
    flops = S * 2 * d * 3 * m
    layer_bytes = touched * 3 * d * m * 2 + w.T * d * 2 * 2 + w.E * d * 2
    roof_ms = max(flops / (pk["bf16_tflops"] * 1e12), layer_bytes / (pk["hbm_gbs"] * 1e9)) * 1e3

    # end to end through the public API with host buffers (no graph), run as a serving
    # loop runs it: every step copies its tokens in from pinned host memory and its
    # outputs back, and the copies of steps i + 1 and i - 1 overlap step i's forward
    # (two device buffer sets, one stream per copy direction).  Timed from the first
    # input copy to the last output copy.
    e2e_ms = max_over_ranks(pipelined_e2e(st, stream, args.steps), ws_n) / args.steps
    e2e_value = ws_n * w.T / (e2e_ms / 1e3)
    nbytes = w.T * w.d * st["u"].element_size()
    del graph

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) tokens)",
        "config": {"workload": w.name, "tokens": w.T, "hidden": w.d, "experts": w.E,
                   "expert_ffn": w.m, "top_k": w.k, "skip_rate": rate,
                   "skip_of": w.skip_of, "router_bias": w.bias, "tau": st["tau"],
                   "parallelism": "replicas" if ws_n > 1 else "single",
                   "launch": "forward captured in one CUDA graph, replayed per step",
                   "l2": "flushed before each timed step (256 MiB write), flush untimed"},
        "workload_stats": {"realised_skip": ss["skipped"] / (w.T * w.k), "kept_slots": S,
                           "touched_experts": touched, "tables": st["tables"],
                           "step_ms": spread},
        "roofline": {"bound": "hbm", "achieved": k_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": k_gbs / pk["hbm_gbs"],
                     "traffic": profiled_traffic(w.name, "fused" if fused else "gateup", rate),
                     "kernel": kname, "algorithmic_bytes": k_bytes, "kernel_ms": k_ms,
                     "algorithmic": "touched experts' weights + X in + Y out",
                     "bytes_incl_intermediates": k_bytes_incl,
                     "frac_incl_intermediates": k_gbs_incl / pk["hbm_gbs"],
                     "peak_source": pk["source"]},
        "kernels": {
            "down": ({"fused": True} if fused else
                     {"achieved_gbs": dn_gbs, "frac": dn_gbs / pk["hbm_gbs"], "kernel_ms": dn_ms,
                      "algorithmic_bytes": dn_bytes}),
            "layer": {"roofline_ms": roof_ms, "frac_of_roofline": roof_ms / ms_step,
                      "tensor_frac": flops / (ms_step / 1e3) / (pk["bf16_tflops"] * 1e12),
                      "flops": flops, "bytes": layer_bytes}},
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
                "d2h_bytes_per_step": nbytes,
                "launch": "plain API calls, no graph; each step's input and output copies "
                          "overlap the neighbouring steps' forwards (two buffer sets, one "
                          "stream per copy direction)", "l2": "no flush: each step streams "
                          "the touched experts' weights, several times the L2"},
        "gpu_launches": KERNELS_PER_FORWARD[fused] * args.steps,
    }
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, st, rate)
    return out


# ------------------------------------------------------------ decode workload
def setup_decode(w, device, n_layers=None):
    """48 independently seeded layers (their weights exceed L2 many times
    over), tables for all of them from one ace_build_tables call (timed), a
    threshold per layer from a 4096-token synthetic pool (quantile mapping),
    and the decode tokens of every layer."""
    from token_dynamic_expert_b200 import ace
    nl = w.layers if n_layers is None else n_layers
    layers = [workloads.make_layer(w, seed=1000 + l, device=device) for l in range(nl)]
    structs = [ace.make_layer(L["gamma"], L["wr"], L["wg"], L["wu"], L["wd"], w.k,
                              router_bias=L["bias"]) for L in layers]
    a_gsp = torch.empty(nl, w.E, dtype=torch.float32, device=device)
    a_rcr = torch.empty_like(a_gsp)
    amax = torch.empty_like(a_gsp)
    sigma = torch.empty(nl, w.E, 3, dtype=torch.float32, device=device)
    tws = ace.alloc_workspace(ace.ace_tables_workspace_size(structs[0]), device)
    ace.ace_build_tables(structs[:1], a_gsp[:1], a_rcr[:1], amax[:1], tws, sigma=sigma[:1])
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    ace.ace_build_tables(structs, a_gsp, a_rcr, amax, tws, sigma=sigma)
    t1.record()
    torch.cuda.synchronize()
    tables_ms = t0.elapsed_time(t1)
    code, flags = ace.ace_read_status(tws)
    if code != ace.ACE_OK:
        raise RuntimeError("table build status %s" % ace.ace_status_str(code))
    del tws
    full = [ace.make_layer(L["gamma"], L["wr"], L["wg"], L["wu"], L["wd"], w.k, amax=amax[l],
                           router_bias=L["bias"]) for l, L in enumerate(layers)]
    pool = max(w.pool, 1)
    pws = ace.alloc_workspace(ace.ace_workspace_size(full[0], pool), device)
    score = torch.empty(pool, w.k, dtype=torch.float32, device=device)
    n_skip = int(np.floor(w.skip * pool * w.k + 0.5))
    # threshold construction: per layer, the pool's scores and the quantile
    # mapping of the skip count, both on the device (timed)
    pools = [workloads.make_tokens(w, T=pool, token_seed=2000 + l, device=device)
             for l in range(nl)]
    tws = ace.alloc_workspace(ace.ace_tau_workspace_size(), device)
    taus_dev = torch.empty(nl, dtype=torch.float32, device=device)
    for rep in range(2):  # the first pass warms up; the second is timed
        t0.record()
        for l in range(nl):
            ace.ace_moe_scores(full[l], pools[l], score, pws)
            ace.ace_tau_quantile(score, n_skip, taus_dev[l:l + 1], tws)
        t1.record()
        torch.cuda.synchronize()
    threshold_ms = t0.elapsed_time(t1)
    taus = [float(t) for t in taus_dev.cpu().tolist()]
    del pws, pools
    us = [workloads.make_tokens(w, T=w.T, token_seed=5000 + l, device=device) for l in range(nl)]
    ys = [torch.empty_like(x) for x in us]
    ws = ace.alloc_workspace(ace.ace_workspace_size(full[0], max(w.T, 1)), device)
    return dict(layers=layers, L=full, taus=taus, u=us, y=ys, ws=ws, amax=amax,
                tables_ms=tables_ms, threshold_ms=threshold_ms, n_layers=nl)


DECODE_PHASES = ["start", "x ready", "barrier 1", "slots", "gate/up done", "barrier 2", "end",
                 "rms sum (token 0)"]


def decode_phases(st, w, stream, reps=5):
    """The decode kernel's per-CTA phase stamps (the debug trace of
    ace_moe_forward), layer 0, L2 flushed before each of `reps` launches:
    median over CTAs of each stamp, in microseconds from the first CTA's
    start, from the last launch."""
    from token_dynamic_expert_b200 import ace
    import ctypes
    dev = st["u"][0].device
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    tr = torch.zeros(nsm, 8, dtype=torch.int64, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            flush.fill_(1)
            dbg = ace.ace_debug_out(trace=ctypes.c_void_p(tr.data_ptr()))
            ace.ace_moe_forward(st["L"][0], st["u"][0], st["taus"][0], st["y"][0], st["ws"],
                                dbg=dbg, stream=stream)
        stream.synchronize()
    t = tr.cpu().numpy().astype(np.float64)
    rel = (t - t[:, 0].min()) / 1e3
    return {n: round(float(np.median(rel[:, i])), 2) for i, n in enumerate(DECODE_PHASES)}


def run_decode(args, w, ws_n, rank, local):
    from token_dynamic_expert_b200 import ace
    dev = torch.device("cuda", local)
    st = setup_decode(w, dev, n_layers=args.layers)
    nl = st["n_layers"]
    stream = torch.cuda.Stream(dev)
    # kept slots and distinct experts per layer (one untimed pass)
    touched, kept, skipped = [], [], 0
    for l in range(nl):
        dbg = ace.DebugOut(w.T, w.k, w.E, dev)
        ace.ace_moe_forward(st["L"][l], st["u"][l], st["taus"][l], st["y"][l], st["ws"], dbg=dbg.c)
        off = dbg.expert_offsets.cpu().numpy()
        touched.append(int((np.diff(off) > 0).sum()))
        kept.append(int(dbg.n_kept.item()))
        skipped += int((dbg.keep == 0).sum().item())
    code, flags = ace.ace_read_status(st["ws"])
    if code != ace.ACE_OK:
        raise RuntimeError("device status %s flags %#x" % (ace.ace_status_str(code), flags))

    def step():
        for l in range(nl):
            ace.ace_moe_forward(st["L"][l], st["u"][l], st["taus"][l], st["y"][l], st["ws"],
                                stream=stream)

    # the 48 layer forwards captured once in a CUDA graph, replayed per step
    # (plain launches are bound by the host's launch rate at ~4 us a kernel)
    with torch.cuda.stream(stream):
        step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        for _ in range(args.warmup):
            graph.replay()
    stream.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(ws_n)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        for i in range(args.steps):
            evs[i][0].record(stream)
            graph.replay()
            evs[i][1].record(stream)
        stream.synchronize()
    barrier(ws_n)
    del graph
    t_steps = [a.elapsed_time(b) for a, b in evs]
    spread = step_spread(t_steps, w.name)
    value, total_ms = replica_throughput(ws_n, args.steps, nl * w.T, sum(t_steps))
    ms_step = total_ms / args.steps
    code, flags = ace.ace_read_status(st["ws"], stream=stream)
    if code != ace.ACE_OK:
        raise RuntimeError("device status %s flags %#x" % (ace.ace_status_str(code), flags))
    # the decode kernel alone, per layer, events recorded by the library
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nl)]
    with torch.cuda.stream(stream):
        for l in range(nl):
            ace.ace_moe_forward(st["L"][l], st["u"][l], st["taus"][l], st["y"][l], st["ws"],
                                dbg=ace.timing_debug(*kev[l]), stream=stream)
        stream.synchronize()
    k_ms = sum(e[0].elapsed_time(e[2]) for e in kev)
    pk = peaks()
    ebytes = 3 * w.d * w.m * 2
    surv = sum(touched) * ebytes
    router = nl * w.E * w.d * 2
    kernel_gbs = (surv + router) / (k_ms / 1e3) / 1e9
    step_gbs = (surv + router) / (ms_step / 1e3) / 1e9
    phases = decode_phases(st, w, stream) if args.trace else None
    # e2e: host tokens in, host outputs back, every layer, plain API calls: one copy of
    # all layers' inputs in and one of their outputs back per step (the layers' buffers
    # side by side), the layer forwards between them on the same stream
    u_all = torch.stack(list(st["u"]))
    y_all = torch.empty_like(u_all)
    u_host = u_all.cpu().pin_memory()
    y_host = torch.empty_like(u_host).pin_memory()
    e2e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps + 1)]
    with torch.cuda.stream(stream):
        for i in range(args.steps + 1):   # the first step warms the path up
            e2e[i][0].record(stream)
            u_all.copy_(u_host, non_blocking=True)
            for l in range(nl):
                ace.ace_moe_forward(st["L"][l], u_all[l], st["taus"][l], y_all[l], st["ws"],
                                    stream=stream)
            y_host.copy_(y_all, non_blocking=True)
            e2e[i][1].record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e[1:]), ws_n)
    nbytes = nl * w.T * w.d * 2
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s (per MoE layer, mean of %d layers)" % nl,
        "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) tokens)",
        "config": {"workload": w.name, "tokens_per_step": w.T, "layers": nl, "hidden": w.d,
                   "experts": w.E, "expert_ffn": w.m, "top_k": w.k, "skip_rate": w.skip,
                   "tau": "per layer, quantile of a %d-token pool" % w.pool,
                   "realised_skip": skipped / (nl * w.T * w.k),
                   "mean_kept_slots": float(np.mean(kept)),
                   "mean_surviving_experts": float(np.mean(touched)),
                   "us_per_layer": ms_step * 1e3 / nl,
                   "parallelism": "replicas" if ws_n > 1 else "single", "step_ms": spread,
                   "launch": "%d layer forwards per step, one CUDA graph" % nl,
                   "l2": "weights of %d layers (%.1f GB) exceed L2; no flush" % (
                       nl, nl * 3 * w.E * w.d * w.m * 2 / 1e9)},
        "roofline": {"bound": "hbm", "achieved": kernel_gbs, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": kernel_gbs / pk["hbm_gbs"], "traffic": None,
                     "kernel": "k_decode (surviving experts' weights + router)",
                     "algorithmic_bytes": (surv + router) / nl, "kernel_ms": k_ms / nl,
                     "peak_source": pk["source"]},
        "kernels": {"step": {"achieved_gbs": step_gbs, "frac": step_gbs / pk["hbm_gbs"]},
                    "tables": {"layers": nl, "experts": w.E, "ms": st["tables_ms"],
                               "ms_per_layer": st["tables_ms"] / nl,
                               "includes": "GSP Grams, power iteration (sigma, 200 steps), RCR"},
                    **({"decode_phases_us": phases} if phases else {}),
                    "thresholds": {"layers": nl, "pool_tokens": max(w.pool, 1),
                                   "ms": st["threshold_ms"],
                                   "includes": "per layer: ace_moe_scores over the pool, "
                                               "ace_tau_quantile (radix select)"}},
        "clocks": clk.summary(),
        "e2e": {"value": ws_n * args.steps * nl * w.T / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                "launch": "plain API calls, no graph; one copy of all layers' inputs in "
                          "and one of their outputs back per step"},
        "gpu_launches": KERNELS_PER_DECODE_LAYER * nl * args.steps,
    }


def run_stack(args, w, ws_n, rank, local):
    """The 48 layers chained through ace_moe_stack_forward: one step is one
    pass of T tokens through every layer (a per-token latency of the MoE
    layers), captured once in a CUDA graph and replayed per step."""
    from token_dynamic_expert_b200 import ace
    dev = torch.device("cuda", local)
    st = setup_decode(w, dev, n_layers=args.layers)
    nl = st["n_layers"]
    stream = torch.cuda.Stream(dev)
    u, y = st["u"][0], torch.empty_like(st["u"][0])
    ws = ace.alloc_workspace(ace.ace_stack_workspace_size(st["L"], w.T), dev)
    # the chain's own routing, layer by layer (untimed): surviving experts
    lws = ace.alloc_workspace(ace.ace_workspace_size(st["L"][0], w.T), dev)
    x, touched, kept = u, [], []
    for l in range(nl):
        dbg = ace.DebugOut(w.T, w.k, w.E, dev)
        out = torch.empty_like(u)
        ace.ace_moe_forward(st["L"][l], x, st["taus"][l], out, lws, dbg=dbg.c)
        off = dbg.expert_offsets.cpu().numpy()
        touched.append(int((np.diff(off) > 0).sum()))
        kept.append(int(dbg.n_kept.item()))
        x = out
    ace.ace_moe_stack_forward(st["L"], u, st["taus"], y, ws, stream=stream)
    stream.synchronize()
    if not torch.equal(y, x):
        raise RuntimeError("stack output differs from the layer-by-layer chain")
    with torch.cuda.stream(stream):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            ace.ace_moe_stack_forward(st["L"], u, st["taus"], y, ws, stream=stream)
        for _ in range(args.warmup):
            g.replay()
    stream.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(ws_n)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        for i in range(args.steps):
            evs[i][0].record(stream)
            g.replay()
            evs[i][1].record(stream)
        stream.synchronize()
    barrier(ws_n)
    t_steps = [a.elapsed_time(b) for a, b in evs]
    spread = step_spread(t_steps, w.name)
    value, total_ms = replica_throughput(ws_n, args.steps, w.T, sum(t_steps))
    ms_step = total_ms / args.steps
    code, flags = ace.ace_read_status(ws, stream=stream)
    if code != ace.ACE_OK:
        raise RuntimeError("device status %s flags %#x" % (ace.ace_status_str(code), flags))
    del g
    pk = peaks()
    surv = sum(touched) * 3 * w.d * w.m * 2
    router = nl * w.E * w.d * 2
    gbs = (surv + router) / (ms_step / 1e3) / 1e9
    # e2e: host tokens in, host outputs back, the plain API call
    u_host = u.cpu().pin_memory()
    y_host = torch.empty_like(u_host).pin_memory()
    e2e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            e2e[i][0].record(stream)
            u.copy_(u_host, non_blocking=True)
            ace.ace_moe_stack_forward(st["L"], u, st["taus"], y, ws, stream=stream)
            y_host.copy_(y, non_blocking=True)
            e2e[i][1].record(stream)
        stream.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e), ws_n)
    nbytes = w.T * w.d * 2
    return {
        "metric": METRIC, "value": value,
        "unit": "tokens/s (through all %d chained MoE layers)" % nl,
        "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) tokens)",
        "config": {"workload": w.name, "tokens_per_step": w.T, "layers": nl, "hidden": w.d,
                   "experts": w.E, "expert_ffn": w.m, "top_k": w.k, "skip_rate": w.skip,
                   "tau": "per layer, quantile of a %d-token pool" % w.pool,
                   "mean_kept_slots": float(np.mean(kept)),
                   "mean_surviving_experts": float(np.mean(touched)),
                   "us_per_layer": ms_step * 1e3 / nl, "tpot_proxy_ms": ms_step,
                   "parallelism": "replicas" if ws_n > 1 else "single", "step_ms": spread,
                   "launch": "ace_moe_stack_forward captured in one CUDA graph",
                   "l2": "weights of %d layers (%.1f GB) exceed L2; no flush" % (
                       nl, nl * 3 * w.E * w.d * w.m * 2 / 1e9)},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / pk["hbm_gbs"], "traffic": None,
                     "kernel": "k_decode x %d layers (whole step)" % nl,
                     "algorithmic_bytes": surv + router, "kernel_ms": ms_step,
                     "peak_source": pk["source"]},
        "clocks": clk.summary(),
        "e2e": {"value": ws_n * args.steps * w.T / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                "launch": "plain API call per step"},
        "gpu_launches": (KERNELS_PER_DECODE_LAYER * nl + 1) * args.steps,
    }


# ---------------------------------------------------------- CPU baselines
def _oracle_inputs(st):
    """Host copies in the oracle's input types (converted once, untimed)."""
    def conv(v):
        if not torch.is_tensor(v):
            return v
        v = v.detach().cpu()
        return np.ascontiguousarray(v.float().numpy())
    layer = {k: conv(v) for k, v in st["layer"].items()}
    amax = st["amax"].cpu().numpy().astype(np.float32)
    u = np.ascontiguousarray(st["u"].detach().cpu().float().numpy().astype(np.float64))
    return layer, u, amax


def oracle_pass_size(layer, u, tau, amax, budget_s):
    """Tokens per oracle pass: the whole batch, or the prefix of it that the
    oracle finishes in about budget_s seconds (from a 4-token probe)."""
    import oracle
    t0 = time.perf_counter()
    oracle.moe_forward(layer, u[:4], tau, amax, amax)
    per_tok = (time.perf_counter() - t0) / 4
    return int(max(4, min(u.shape[0], budget_s / max(per_tok, 1e-9))))


def oracle_passes(layer, u, tau, amax, n, passes, warm=1):
    """Seconds of each of `passes` oracle forwards over the first n tokens,
    after `warm` untimed ones.  Both oracle timings of this script (the
    cpu_baseline leg and the reference arm) run through here, under one
    condition: torch's own CPU thread pool is held at one thread meanwhile,
    so the host cores belong to the oracle's threads."""
    import oracle
    nt = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        for _ in range(warm):
            oracle.moe_forward(layer, u[:n], tau, amax, amax)
        times = []
        for _ in range(passes):
            t0 = time.perf_counter()
            oracle.moe_forward(layer, u[:n], tau, amax, amax)
            times.append(time.perf_counter() - t0)
    finally:
        torch.set_num_threads(nt)
    return times


def cpu_baseline(w, st, rate, target_s=12.0, pass_budget_s=6.0):
    """The oracle as it stands on the host cores, on a bounded sample of the
    same workload: one warm-up pass, then whole passes over the batch's
    tokens (or the prefix that fits pass_budget_s) until about target_s
    seconds of CPU work."""
    import oracle
    layer, u, amax = _oracle_inputs(st)
    n = oracle_pass_size(layer, u, st["tau"], amax, pass_budget_s)
    t1 = oracle_passes(layer, u, st["tau"], amax, n, 1, warm=1)[0]
    passes = int(max(1, min(64, target_s / max(t1, 1e-9)) - 1))
    times = [t1] + oracle_passes(layer, u, st["tau"], amax, n, passes, warm=0)
    dt = sum(times)
    return {"value": len(times) * n / dt, "unit": "tokens/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": "%d passes over the first %d of the batch's %d tokens after one warm-up "
                      "pass (fp64 forward incl. routing, mask and combine), %.1f s; pass "
                      "%.3f-%.3f s; torch CPU threads held at 1" % (
                          len(times), n, w.T, dt, min(times), max(times))}


def run_reference(args, w, rate):
    """The reference arm: the fp64 CPU oracle, each step one pass over a
    bounded sample of the batch.  The untimed set-up (layer, tables, tau)
    is the GPU arm's own, so both arms see the same workload."""
    import oracle
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else None
    if dev is None:
        layer = workloads.make_layer(w)
        u = workloads.make_tokens(w)
        amax = np.ones(w.E, dtype=np.float32)
        tau = 0.0
        layer = {k: (v.float().numpy() if torch.is_tensor(v) else v) for k, v in layer.items()}
        u = u.double().numpy()
    else:
        st = setup_prefill(w, rate, dev)
        layer, u, amax = _oracle_inputs(st)
        tau = st["tau"]
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = oracle_pass_size(layer, u, tau, amax, budget)
    times = oracle_passes(layer, u, tau, amax, n, args.steps, warm=args.warmup)
    dt = sum(times)
    val = args.steps * n / dt
    unit = "tokens/s"
    sample = "%d of %d tokens per step (one oracle pass), %d warm-up passes; pass %.3f-%.3f s; " \
             "torch CPU threads held at 1" % (n, w.T, args.warmup, min(times), max(times))
    if w.name.startswith("stack"):  # one layer timed; the chain costs layers times as much
        val /= w.layers
        unit = "tokens/s (through all %d chained MoE layers)" % w.layers
        sample += "; one layer timed, the %d-layer rate is its rate / %d" % (w.layers, w.layers)
    config = {"workload": w.name, "tokens": w.T, "hidden": w.d, "experts": w.E,
              "expert_ffn": w.m, "top_k": w.k, "skip_rate": rate, "skip_of": w.skip_of,
              "router_bias": w.bias, "tau": tau,
              "parallelism": "replicas" if args.gpus > 1 else "single",
              "launch": "one oracle pass per step on the host cores",
              "l2": "not applicable: the oracle runs on the host"}
    return {"metric": METRIC, "value": val, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,0.02) weights, N(0,1) tokens)", "impl": "reference",
            "config": config,
            "cpu_baseline": {"value": val, "unit": unit, "kind": "oracle",
                             "cores": oracle.threads(), "sample": sample},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="prefill_1024",
                    choices=["prefill_1024", "prefill_8192_e256", "sweep_4096", "decode_bs1",
                             "decode_bs8", "stack_bs1", "stack_bs8"])
    ap.add_argument("--rate", type=float, default=None, help="override the skip rate")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="decode: number of layers (default: the workload's 48)")
    ap.add_argument("--trace", action="store_true",
                    help="decode: add the decode kernel's phase timeline (debug trace)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    w = workloads.WORKLOADS[args.workload]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        rate = w.skip if args.rate is None else args.rate
        print(json.dumps(run_reference(args, w, rate)), flush=True)
        return

    from token_dynamic_expert_b200 import build as _b  # noqa: F401  (the .so ships prebuilt)
    ws_n, rank, local = dist_setup(args.gpus)
    if args.workload.startswith("decode") or args.workload.startswith("stack"):
        run = run_decode if args.workload.startswith("decode") else run_stack
        out = run(args, w, ws_n, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
        if ws_n > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    rates = [w.skip if args.rate is None else args.rate]
    if args.workload == "sweep_4096" and args.rate is None:
        rates = list(workloads.SWEEP_RATES)
    for rate in rates:
        out = run_ours(args, w, rate, ws_n, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
