"""Benchmark of the multi-precision BCQ GEMV on B200.

Workload: one BCQ weight of the Llama-3.1-8B MLP gate/up shape
(N = 14336 outputs, K = 4096 inputs, group 128, p_H = 4 stored planes) with
synthetic seeded data (bit_gemv_bcq_b200/synth.py).  One step is one call for
every precision p in {2, 3, 4} and batch M in {1, 2, 4, 8, 16}: 15 calls.
Metric: achieved HBM throughput in GB/s over the algorithmic bytes
    N*K*p/8 (planes) + N*G*p*2 (scales) + N*G*2 (offsets) + M*K*2 (x) + M*N*2 (y)
of every call, with microseconds per call reported per (p, M).

Timing: CUDA graphs (one per step, 15 calls) replayed back to back; R
rotating copies of the weights (> 2x L2 in total) so every call streams from
HBM; CUDA events on the launching stream; W warm-up steps; clocks sampled
with nvidia-smi during the timed work.  Per call (`per_call`, `headline_m1`,
`shapes`): graphs of 200 calls cycling through a weight ring, median of 5
replays, programmatic dependent launch as --pdl says (back to back);
`isolated_m1`: one call with PDL off and L2 flushed before it.  `shapes`
covers the other workload shapes: 4096 x 4096 (M = 1), the MLP decode pair
with 0.1 % outlier channels (M = 1), and the 70B-like pair with 8 rows of
per-request precision.  ``e2e`` measures the step's calls through the C
entry point with host buffers (bcq_gemm_host), copies included.  The
`roofline` object is that of the step's dominant kernel (most time per
step), the step aggregate beside it.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload on the host cores.  With torchrun (N > 1 GPUs) every rank runs
an independent replica (no collective on the data path; --mode shard: one
layer split by output rows, an NCCL all-gather of y per call), the timed
region is bracketed by barriers and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_OUT, K_IN, GROUP, P_H = 14336, 4096, 128, 4
PRECISIONS = (2, 3, 4)
BATCHES = (1, 2, 4, 8, 16)
METRIC = "BCQ GEMV µs & HBM GB/s (% of B200 peak) at p=2/3/4, M=1..16, 14336×4096"
WORKLOAD = ("bcq_gemv N=14336 K=4096 g=128 p_H=4; one step = one call per p in {2,3,4} x "
            "M in {1,2,4,8,16} (15 calls), fp16 x/y/scales")
REF_BUDGET_S = 90.0   # host work of one reference-arm run (warm-up and timed steps)
L2_BYTES = 126 * 1024 * 1024


def algo_bytes(N, K, M, p):
    G = K // GROUP
    return N * K * p // 8 + N * G * p * 2 + N * G * 2 + M * K * 2 + M * N * 2


# Sources of the kernels the bench step launches (one-row, pair, four-row and
# mma.sync kernels; the step launches no tcgen05 kernel)
KERNEL_SOURCES = ("bcq_kernels.cu", "bcq_device.cuh", "bcq_pipeline.cuh", "bcq_mma.cuh",
                  "bcq_m1.cuh", "bcq_layout.h")
# CUDA kernel of each launch kind bcq_route_query reports
KERNEL_OF_ROUTE = {"lut_one": "gemv_m1_kernel", "lut_pair": "gemv_lut_kernel<2>",
                   "lut_four": "gemv_lut_kernel<4>", "mma": "gemv_mma_kernel",
                   "mma_mixed": "gemv_mma_kernel<mixed>", "tcgen05": "gemv_umma_kernel"}


def csrc_sha256():
    """Hash of the sources that define the GEMV kernels (recorded DRAM
    traffic is only reported while they are unchanged)."""
    import hashlib
    h = hashlib.sha256()
    src = os.path.join(ROOT, "bit_gemv_bcq_b200", "csrc")
    for f in KERNEL_SOURCES:
        h.update(f.encode())
        with open(os.path.join(src, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu launch list, or None when
    the kernel sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        if t.get("csrc_sha256") != csrc_sha256():
            return None
        return t
    except Exception:
        return None


def recorded_quantizer_insts():
    """Warp instructions per group of the quantiser kernel from the committed
    ncu capture, or None when bcq_quantize.cu changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "quantize_issue.json")) as f:
            t = json.load(f)
        with open(os.path.join(ROOT, "bit_gemv_bcq_b200", "csrc", "bcq_quantize.cu"), "rb") as f:
            h = hashlib.sha256(b"bcq_quantize.cu" + f.read()).hexdigest()
        return t if t.get("source_sha256") == h else None
    except Exception:
        return None


SM_COUNT, SM_SUBPARTITIONS, SM_MAX_MHZ = 148, 4, 1965.0


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------- ranks (N > 1)

def rank_barrier(world):
    """Barrier of all ranks (no-op on one GPU)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device):
    """The largest value over all ranks (the job's time is its slowest
    rank's); `device` is where the process group's backend reduces (cuda for
    NCCL, cpu for gloo)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbps(bytes_per_rank_step, ms_per_step, world):
    """Whole-job throughput: every rank processes its own bytes_per_rank_step
    per step (weak scaling, replicas), in ms_per_step (the max over ranks)."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="bcq_clocks_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, maxs, reasons, powers = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [s.strip() for s in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    maxs.append(float(parts[2]))
                    powers.append(float(parts[3]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "samples": len(sms), "power_w_max": max(powers) if powers else None,
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ GPU arm

CALLS_PER_GRAPH = 200   # calls captured per timing graph
REPLAYS = 5             # timed replays; the median is reported


def weight_bytes(w):
    return w.packed.numel() * 4 + sum(a.numel() * 2 for a in w.alphas.values()) + \
        (w.z.numel() * 2 if w.z is not None else 0) + \
        (sum(v.numel() * 2 for v in w.zq.values()) if w.zq else 0)


def weight_ring(api, base):
    """base and copies of it, more than 2x L2 in all, so that every call
    streams its weights from HBM."""
    per = weight_bytes(base)
    R = max(2, math.ceil(2 * L2_BYTES / per) + 1)
    ring = [base]
    for _ in range(R - 1):
        ring.append(api.BcqWeights(
            packed=base.packed.clone(), alphas={q: a.clone() for q, a in base.alphas.items()},
            z=None if base.z is None else base.z.clone(), N=base.N, K=base.K, p_H=base.p_H,
            row_splits=base.row_splits,
            zq=None if base.zq is None else {q: v.clone() for q, v in base.zq.items()}))
    return ring, per


def run_gpu(args, rank, world, local_rank):
    import torch
    from bit_gemv_bcq_b200 import api, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    prob = synth.make_problem(N_OUT, K_IN, max(BATCHES), seed=args.seed)
    base = api.BcqWeights.from_canonical(prob.planes, prob.alphas, prob.z, device=dev)
    copies, per_copy = weight_ring(api, base)
    R = len(copies)
    x = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).to(dev)
    ys = {M: torch.empty((M, N_OUT), dtype=torch.float16, device=dev) for M in BATCHES}
    cases = [(p, M) for p in PRECISIONS for M in BATCHES]
    if args.cases:
        want = {tuple(int(v) for v in c.split(":")) for c in args.cases.split(",")}
        cases = [(p, M) for p, M in cases if (M, p) in want]
    bytes_step = sum(algo_bytes(N_OUT, K_IN, M, p) for p, M in cases)
    api.set_pdl(args.pdl)
    routes = {(p, M): api.route_query(M, N_OUT, K_IN, p=p) for p, M in cases}
    launches_per_step = sum(len(r) for r in routes.values())

    stream = torch.cuda.Stream(device=dev)
    # eager pass: plans and caches every launch shape before capture
    with torch.cuda.stream(stream):
        for p, M in cases:
            base.gemm(x[:M], p=p, out=ys[M], stream=stream)
    stream.synchronize()
    assert api.device_error(stream) == api.BCQ_OK

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    def us_per_call(fn_calls, ncalls):
        """Median over REPLAYS of one replay of a graph of ncalls calls."""
        g = capture(fn_calls)
        times = []
        with torch.cuda.stream(stream):
            g.replay()
            for _ in range(REPLAYS):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                times.append((a, b))
        stream.synchronize()
        del g
        return statistics.median(a.elapsed_time(b) for a, b in times) * 1000.0 / ncalls

    step_graphs = []
    for r in range(R):
        def step(r=r):
            for i, (p, M) in enumerate(cases):
                copies[(r + i) % R].gemm(x[:M], p=p, out=ys[M], stream=stream)
        step_graphs.append(capture(step))

    def barrier():
        rank_barrier(world)

    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            step_graphs[k % R].replay()
    stream.synchronize()

    # clocks are sampled over all the timed work below (the step, then the
    # per-call timings)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.2)
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for k in range(args.steps):
            step_graphs[k % R].replay()
        t1.record(stream)
    t1.synchronize()
    torch.cuda.synchronize(dev)
    barrier()
    ms_total = t0.elapsed_time(t1)
    del step_graphs
    err = api.device_error(stream)
    if err != api.BCQ_OK:
        raise RuntimeError(f"device error {api.status_string(err)}")
    ms_total = max_over_ranks(ms_total, world, dev)

    # per-call microseconds of each case, back to back: a graph of 200 calls
    # cycling through the weight ring, median of 5 replays
    per_case = []
    for p, M in cases:
        def calls(p=p, M=M):
            for i in range(args.calls):
                copies[i % R].gemm(x[:M], p=p, out=ys[M], stream=stream)
        us = us_per_call(calls, args.calls)
        by = algo_bytes(N_OUT, K_IN, M, p)
        per_case.append({"p": p, "M": M, "us": round(us, 3), "bytes": by,
                         "GBps": round(by / us / 1e3, 1),
                         "kernels": [k for k, _, _ in routes[(p, M)]]})

    # one call alone: programmatic dependent launch off, L2 flushed (a write
    # of 2x L2) before it, CUDA events around that call only
    isolated = None
    if not args.cases:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
        api.set_pdl(0)
        isolated = {"method": "PDL off, L2 flushed before each call, median of 20 calls"}
        for p in PRECISIONS:
            g = capture(lambda p=p: copies[0].gemm(x[:1], p=p, out=ys[1], stream=stream))
            times = []
            with torch.cuda.stream(stream):
                for _ in range(21):
                    flush.fill_(1)
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    g.replay()
                    b.record(stream)
                    times.append((a, b))
            stream.synchronize()
            us = statistics.median(a.elapsed_time(b) for a, b in times[1:]) * 1000.0
            by = algo_bytes(N_OUT, K_IN, 1, p)
            isolated[f"M1p{p}"] = {"us": round(us, 3), "GBps": round(by / us / 1e3, 1)}
            del g
        del flush
        api.set_pdl(args.pdl)
    clocks = sampler.stop()

    # the other workload shapes, same back-to-back method (each on its own
    # weight ring): the attention projection, the MLP down projection (and
    # gate/up) with 0.1 % outlier channels, and the 70B-like shapes with 8 rows
    # of per-request precision
    shapes = None
    if not args.cases:
        shapes = {}
        specs = [("attn_4096x4096_M1", 4096, 4096, 1, False, False),
                 ("mlp_gate_up_14336x4096_M1_outliers", 14336, 4096, 1, True, False),
                 ("mlp_down_4096x14336_M1_outliers", 4096, 14336, 1, True, False),
                 ("70b_28672x8192_M8_mixed", 28672, 8192, 8, False, True),
                 ("70b_8192x28672_M8_mixed", 8192, 28672, 8, False, True)]
        for label, N, K, M, outl, mixed in specs:
            pr = synth.make_problem(N, K, M, seed=args.seed + 4, outliers=outl, mixed=mixed)
            wb = api.BcqWeights.from_canonical(pr.planes, pr.alphas, pr.z, device=dev)
            ring, per = weight_ring(api, wb)
            xs = torch.from_numpy(pr.x.view(np.int16)).view(torch.float16).to(dev)
            yy = torch.empty((M, N), dtype=torch.float16, device=dev)
            entry = {"N": N, "K": K, "M": M, "ring": f"{len(ring)} copies of {per / 2**20:.1f} MiB"}
            for p in ([None] if mixed else PRECISIONS):
                kw = {"p_row": pr.p_row} if mixed else {"p": p}
                with torch.cuda.stream(stream):
                    wb.gemm(xs, out=yy, stream=stream, **kw)
                stream.synchronize()

                def calls(kw=kw):
                    for i in range(args.calls):
                        ring[i % len(ring)].gemm(xs, out=yy, stream=stream, **kw)
                us = us_per_call(calls, args.calls)
                G = K // GROUP
                if mixed:
                    qs = sorted(set(pr.p_row.tolist()))
                    by = N * K * max(qs) // 8 + sum(N * G * q * 2 for q in qs) + N * G * 2 \
                        + M * K * 2 + M * N * 2
                    key = "mixed"
                    entry["p_row"] = [int(v) for v in pr.p_row]
                else:
                    by = algo_bytes(N, K, M, p)
                    key = f"p{p}"
                route = api.route_query(M, N, K, **kw)
                entry[key] = {"us": round(us, 3), "bytes": by, "GBps": round(by / us / 1e3, 1),
                              "launches": [f"{k}:{n}rows:{pl}planes" for k, n, pl in route]}
            shapes[label] = entry
            del ring, wb, xs, yy
            torch.cuda.synchronize(dev)
        shapes["attn_4096x4096_M1"]["context"] = (
            "ABQ-LLM page (GEMV ablation): 6.68 us for a (1,4096)x(4096,4096) W2A8 GEMV "
            "on RTX 3070/4080 -- other hardware, activations quantised to 8 bits; context only")
        assert api.device_error(stream) == api.BCQ_OK

    # an MLP's gate and up projections (same x) stacked into one weight: one
    # call for both (M = 1, 2), against two calls on the separate weights
    stacked = None
    if not args.cases:
        prob_b = synth.make_problem(N_OUT, K_IN, max(BATCHES), seed=args.seed + 1)
        sbase = api.BcqWeights.stack([(prob.planes, prob.alphas, prob.z),
                                      (prob_b.planes, prob_b.alphas, prob_b.z)], device=dev)
        scopies, s_copy = weight_ring(api, sbase)
        ys2 = {M: torch.empty((M, sbase.N), dtype=torch.float16, device=dev) for M in (1, 2)}
        with torch.cuda.stream(stream):
            for M in (1, 2):
                for p in PRECISIONS:
                    sbase.gemm(x[:M], p=p, out=ys2[M], stream=stream)
        stream.synchronize()
        stacked = {"weights": f"2 x {N_OUT} rows (gate and up) x {K_IN}, stacked along N",
                   "l2": f"{len(scopies)} rotating copies of {s_copy / 2**20:.1f} MiB"}
        single = {(c["p"], c["M"]): c["us"] for c in per_case}
        for M in (1, 2):
            for p in PRECISIONS:
                def sone(p=p, M=M):
                    for i in range(args.calls):
                        scopies[i % len(scopies)].gemm(x[:M], p=p, out=ys2[M], stream=stream)
                us = us_per_call(sone, args.calls)
                by = algo_bytes(2 * N_OUT, K_IN, M, p)
                two = 2 * single[(p, M)] if (p, M) in single else None
                stacked[f"M{M}p{p}"] = {"us": round(us, 3), "GBps": round(by / us / 1e3, 1),
                                        "us_two_calls": None if two is None else round(two, 3)}
        del scopies, sbase
        assert api.device_error(stream) == api.BCQ_OK

    # offsets per precision (bcq_gemm_zp): M = 1 at each precision and one
    # two-row launch with two precisions, against the same calls with shared
    # offsets
    zp = None
    if not args.cases:
        rng = np.random.default_rng(args.seed + 3)
        zq = {q: rng.normal(0.0, 0.005, size=prob.z.shape).astype(np.float16) for q in PRECISIONS}
        zbase = api.BcqWeights.from_canonical(prob.planes, prob.alphas, zq, device=dev)
        zcopies = [zbase] + [api.BcqWeights(packed=c.packed, alphas=c.alphas, z=None, N=c.N, K=c.K,
                                            p_H=c.p_H, zq={q: v.clone() for q, v in zbase.zq.items()})
                             for c in copies[1:]]
        zp = {"weights": "the bench weight with one offset array per precision"}
        single = {(c["p"], c["M"]): c["us"] for c in per_case}
        for label, M, pr in [("M1p2", 1, [2]), ("M1p3", 1, [3]), ("M1p4", 1, [4]),
                             ("M2p2p4", 2, [2, 4])]:
            with torch.cuda.stream(stream):
                zbase.gemm(x[:M], p_row=pr, out=ys[M], stream=stream)
            stream.synchronize()

            def zone(M=M, pr=pr):
                for i in range(args.calls):
                    zcopies[i % len(zcopies)].gemm(x[:M], p_row=pr, out=ys[M], stream=stream)
            us = us_per_call(zone, args.calls)
            shared = single.get((pr[0], M)) if len(set(pr)) == 1 else None
            zp[label] = {"us": round(us, 3), "us_shared_offsets": shared}
        del zcopies, zbase
        assert api.device_error(stream) == api.BCQ_OK

    result = {"ms_total": ms_total, "bytes_step": bytes_step, "R": R,
              "per_copy_bytes": per_copy, "launches_per_step": launches_per_step,
              "per_case": per_case, "clocks": clocks, "stacked": stacked,
              "per_precision_offsets": zp, "shapes": shapes, "isolated": isolated}

    # end to end through bcq_gemm_host: pinned host x and y, copies inside
    # the timed region.  Calls alternate between two streams, each with its
    # own staging buffers, output buffers and workspace, so one call's
    # copies overlap the other's kernels (a pipelined caller).
    if not args.profile:
        x_host = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).pin_memory()
        streams = [stream, torch.cuda.Stream(device=dev)]
        y_host = [{M: torch.empty((M, N_OUT), dtype=torch.float16).pin_memory() for M in BATCHES}
                  for _ in streams]
        x_dev = [torch.empty_like(x) for _ in streams]
        y_dev = [{M: torch.empty((M, N_OUT), dtype=torch.float16, device=dev) for M in BATCHES}
                 for _ in streams]
        # the first M rows of the staging buffers, as views made once (a
        # caller with fixed buffers slices them once, not per call)
        x_host_m = {M: x_host[:M] for M in BATCHES}
        x_dev_m = [{M: xd[:M] for M in BATCHES} for xd in x_dev]
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        h2d = sum(M * K_IN * 2 for _, M in cases)
        d2h = sum(M * N_OUT * 2 for _, M in cases)

        def e2e_step(k):
            for i, (p, M) in enumerate(cases):
                j = (k * len(cases) + i) % 2
                api.gemm_host(x_host_m[M], copies[(k + i) % R], y_host[j][M], x_dev_m[j][M],
                              y_dev[j][M], p=p, stream=streams[j])

        for k in range(2):
            e2e_step(k)
        for st_ in streams:
            st_.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(streams[0])
        streams[1].wait_event(a)
        for k in range(e2e_steps):
            e2e_step(k)
        joined = torch.cuda.Event()
        joined.record(streams[1])
        streams[0].wait_event(joined)
        b.record(streams[0])
        b.synchronize()
        e2e_ms = a.elapsed_time(b)
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        assert api.device_error(streams[0]) == api.BCQ_OK and api.device_error(streams[1]) == api.BCQ_OK
        # (outside the timed region) the host path gives the device path's bits
        for p, M in cases:
            api.gemm_host(x_host[:M], copies[0], y_host[0][M], x_dev[0][:M], y_dev[0][M], p=p,
                          stream=streams[0])
            copies[0].gemm(x[:M], p=p, out=ys[M], stream=streams[0])
            streams[0].synchronize()
            if not torch.equal(y_host[0][M], ys[M].cpu()):
                raise RuntimeError(f"e2e output differs from the device path (p={p}, M={M})")
        result["e2e"] = {"ms": e2e_ms, "steps": e2e_steps, "h2d": h2d, "d2h": d2h}
    return result


def run_sharded(args, rank, world, local_rank):
    """One 14336 x 4096 layer split by output rows over the ranks: each rank
    packs its rows, runs the step's 15 calls on them and all-gathers y after
    every call (NCCL; the only collective).  Steps are CUDA graphs over a ring
    of copies of the rank's rows; the time is the max over ranks; `value` is
    the whole layer's algorithmic bytes per step over that time (strong
    scaling: the total work is fixed)."""
    import torch
    from bit_gemv_bcq_b200 import api, shard, synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    prob = synth.make_problem(N_OUT, K_IN, max(BATCHES), seed=args.seed)
    sw = shard.ShardedBcqWeights.from_canonical(prob.planes, prob.alphas, prob.z, world, rank,
                                                device=dev)
    ring, per = weight_ring(api, sw.local)
    copies = [shard.ShardedBcqWeights(w, N_OUT, sw.r0, sw.r1, world, rank) for w in ring]
    x = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).to(dev)
    cases = [(p, M) for p in PRECISIONS for M in BATCHES]
    bytes_step = sum(algo_bytes(N_OUT, K_IN, M, p) for p, M in cases)
    api.set_pdl(args.pdl)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for p, M in cases:
            copies[0].gemm(x[:M], p=p, stream=stream)
    stream.synchronize()
    graphs = []
    for r in range(len(copies)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i, (p, M) in enumerate(cases):
                copies[(r + i) % len(copies)].gemm(x[:M], p=p, stream=stream)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            graphs[k % len(graphs)].replay()
    stream.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.2)
    rank_barrier(world)
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for k in range(args.steps):
            graphs[k % len(graphs)].replay()
        t1.record(stream)
    t1.synchronize()
    torch.cuda.synchronize(dev)
    rank_barrier(world)
    clocks = sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    del graphs
    assert api.device_error(stream) == api.BCQ_OK
    peak, peak_kind = measured_peaks()
    ms_step = ms / args.steps
    value = bytes_step / (ms_step * 1e-3) / 1e9
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "bcq_gemv N=14336 K=4096 g=128 p_H=4, split by output rows "
                                   f"over {world} ranks; one step = one call per p in {{2,3,4}} x "
                                   "M in {1,2,4,8,16} + an all-gather of y after each",
                       "l2": f"{len(ring)} rotating copies of this rank's {per / 2**20:.1f} MiB",
                       "parallelism": f"column-parallel x{world} (NCCL all-gather)"},
            "roofline": {"bound": "hbm", "achieved": round(value / world, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(value / world / peak, 4),
                         "peak_kind": peak_kind, "traffic": None,
                         "kernel": "per GPU: the rank's rows of every call of the step"},
            "gpu_launches": sum(len(api.route_query(M, sw.r1 - sw.r0, K_IN, p=p))
                                for p, M in cases) * args.steps,
            "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_quantizer(args, dev, rows=N_OUT):
    """The offline quantiser (bcq_quantize) on one fp16 weight of `rows` x
    K_IN: p_L = 2 -> p_H = 4, 20 refinement rounds.  Each timed call is
    preceded by an L2 flush (a write of 2x L2) outside its events."""
    import torch
    from bit_gemv_bcq_b200 import api, synth
    w16 = synth.make_weights(rows, K_IN, seed=args.seed + 7)
    w = torch.from_numpy(w16.view(np.int16)).view(torch.float16).to(dev)
    G = K_IN // GROUP
    planes = torch.empty((P_H, rows, K_IN // 32), dtype=torch.int32, device=dev)
    alphas = {p: torch.empty((rows, G, p), dtype=torch.float16, device=dev) for p in PRECISIONS}
    z = torch.empty((rows, G), dtype=torch.float16, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    arr = api._alpha_array(alphas)

    zq = {p: torch.empty((rows, G), dtype=torch.float16, device=dev) for p in PRECISIONS}
    zarr = api._alpha_array(zq, "z")

    def call(per_precision=False):
        if per_precision:
            st = api.lib().bcq_quantize_zp(api._ptr(w), rows, K_IN, 2, P_H, 20, api._ptr(planes),
                                           arr, zarr, None, api._stream(stream))
        else:
            st = api.lib().bcq_quantize(api._ptr(w), rows, K_IN, 2, P_H, 20, api._ptr(planes), arr,
                                        api._ptr(z), None, api._stream(stream))
        if st != api.BCQ_OK:
            raise api.BcqError(st, "bcq_quantize")

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    stream.synchronize()
    reps = 10
    ms = 0.0
    for _ in range(reps):
        with torch.cuda.stream(stream):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
        b.synchronize()
        ms += a.elapsed_time(b)
    ms /= reps
    # the per-precision-offset variant (bcq_quantize_zp), same method
    with torch.cuda.stream(stream):
        call(True)
    ms_zp = 0.0
    for _ in range(reps):
        with torch.cuda.stream(stream):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call(True)
            b.record(stream)
        b.synchronize()
        ms_zp += a.elapsed_time(b)
    ms_zp /= reps
    assert api.device_error(stream) == api.BCQ_OK
    groups = rows * G
    out = {"workload": f"bcq_quantize fp16 {rows}x{K_IN}, g=128, p_L=2 -> p_H=4, 20 rounds "
                       f"({groups} groups, a quarter warp each)",
           "ms": round(ms, 4), "groups_per_s": round(groups / (ms * 1e-3), 1),
           "weights_GBps": round(rows * K_IN * 2 / (ms * 1e-3) / 1e9, 2),
           "launches_per_call": 1, "reps": reps, "l2": "flushed before every call",
           "ms_per_precision_offsets": round(ms_zp, 4)}
    # issue-bound fp64/integer code: achieved warp instructions per second
    # (ncu's count per group x groups / event time) against the issue peak
    # of 148 SMs x 4 schedulers x one warp instruction per cycle at 1965 MHz
    rec = recorded_quantizer_insts()
    peak = SM_COUNT * SM_SUBPARTITIONS * SM_MAX_MHZ * 1e6
    if rec is not None:
        ach = rec["warp_insts_per_group"] * groups / (ms * 1e-3)
        out["roofline"] = {"bound": "alu", "achieved": round(ach / 1e9, 1), "peak": round(peak / 1e9, 1),
                           "unit": "G warp-instructions/s", "frac": round(ach / peak, 4),
                           "insts_per_group": rec["warp_insts_per_group"], "source": rec["source"]}
    return out


def run_quantizer_oracle(seed, n_groups=1024):
    """The fp64 quantiser oracle on a sample of groups of the same weight."""
    from oracle import quantizer as Q
    from bit_gemv_bcq_b200 import synth
    w16 = synth.make_weights(N_OUT, K_IN, seed=seed + 7)
    rng = np.random.default_rng(seed + 8)
    G = K_IN // GROUP
    picks = rng.choice(N_OUT * G, n_groups, replace=False)
    sub = np.stack([w16[q // G, (q % G) * GROUP:(q % G + 1) * GROUP] for q in picks])
    t0 = time.perf_counter()
    Q.quantize_groups(sub.astype(np.float64), 2, P_H, 20)
    dt = time.perf_counter() - t0
    return {"groups_per_s": round(n_groups / dt, 2), "cores": 1, "kind": "oracle",
            "sample": f"{n_groups} random groups of the same weight ({dt:.1f} s)"}


# ------------------------------------------------------------- CPU oracle arm

def run_oracle_sample(seed, rows_per_call, prob=None):
    """The fp64 oracle on a bounded sample: `rows_per_call` output rows of each
    of the 15 calls.  Returns (seconds, algorithmic bytes of the sample, threads)."""
    import oracle
    from bit_gemv_bcq_b200 import synth
    if prob is None:
        prob = synth.make_problem(N_OUT, K_IN, max(BATCHES), seed=seed)
    rng = np.random.default_rng(seed + 1)
    rows = np.sort(rng.choice(N_OUT, rows_per_call, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    for p in PRECISIONS:
        for M in BATCHES:
            oracle.gemm(prob.x[:M], prob.planes, prob.alphas, prob.z, p=p, rows=rows)
    dt = time.perf_counter() - t0
    frac = rows_per_call / N_OUT
    by = sum(algo_bytes(N_OUT, K_IN, M, p) for p in PRECISIONS for M in BATCHES) * frac
    return dt, by, oracle.num_threads()


def reference_arm(args):
    """The oracle as the reference arm: W untimed and exactly K timed steps, each
    step the 15 calls of the workload on a sample of output rows.  The sample is
    sized so that the whole run costs about REF_BUDGET_S seconds of host work:
    a step costs a fixed part (15 oracle calls) plus a part per sampled row,
    both taken from two calibration samples."""
    from bit_gemv_bcq_b200 import synth
    prob = synth.make_problem(N_OUT, K_IN, max(BATCHES), seed=args.seed)
    t_lo = run_oracle_sample(args.seed, 16, prob)[0]
    t_hi = run_oracle_sample(args.seed, 256, prob)[0]
    per_row = max((t_hi - t_lo) / 240, 1e-9)
    fixed = max(t_lo - 16 * per_row, 0.0)
    per_step = REF_BUDGET_S / (args.steps + args.warmup)
    rows = int((per_step - fixed) / per_row) // 16 * 16
    rows = max(16, min(args.cpu_rows, 2048, rows))
    for k in range(args.warmup):
        run_oracle_sample(args.seed + 1 + k, rows, prob)
    secs, by, thr = 0.0, 0.0, 1
    for k in range(args.steps):
        s, b, thr = run_oracle_sample(args.seed + 1 + args.warmup + k, rows, prob)
        secs += s
        by += b
    gbps = by / secs / 1e9
    return {"metric": METRIC, "value": round(gbps, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "parallelism": "single process, host cores"},
            "cpu_baseline": {"value": round(gbps, 4), "unit": "GB/s", "cores": thr,
                             "kind": "oracle",
                             "sample": f"{rows} of {N_OUT} output rows of each of the 15 calls "
                                       f"per step, {args.steps} timed steps after "
                                       f"{args.warmup} untimed"},
            "e2e": {"value": round(gbps, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="bcq", choices=["bcq", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-rows", type=int, default=14336,
                    help="output rows per call in the oracle's timed sample")
    ap.add_argument("--cpu-reps", type=int, default=4,
                    help="repetitions of the oracle's sample (about 10-30 s of CPU work)")
    ap.add_argument("--cases", default="",
                    help="restrict the step to these M:p pairs (profiling only), e.g. 1:2,1:3")
    ap.add_argument("--pdl", type=int, default=2, choices=[0, 1, 2],
                    help="bcq_set_pdl mode for the GEMV launches (2: weights may stream "
                         "while the previous kernel drains; no kernel of the step writes them)")
    ap.add_argument("--calls", type=int, default=CALLS_PER_GRAPH,
                    help="calls per per-call timing graph (fewer for profiler runs)")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "shard"],
                    help="N > 1 GPUs: independent replicas of the workload (weak scaling), "
                         "or one layer split by output rows over the ranks with an NCCL "
                         "all-gather of y per call (strong scaling)")
    ap.add_argument("--profile", action="store_true",
                    help="GPU timing only (no e2e or CPU legs), for profiler runs")
    ap.add_argument("--quantizer-only", type=int, default=0, metavar="ROWS",
                    help="only time the offline quantiser on ROWS x 4096 weights (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(reference_arm(args)), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.quantizer_only:
        torch.cuda.set_device(local_rank)
        q = run_quantizer(args, torch.device("cuda", local_rank), rows=args.quantizer_only)
        if rank == 0:
            print(json.dumps({"quantizer": q}), flush=True)
        return 0
    if args.mode == "shard":
        return run_sharded(args, rank, world, local_rank)
    res = run_gpu(args, rank, world, local_rank)
    quant = run_quantizer(args, torch.device("cuda", local_rank)) if not args.cases else None

    peak, peak_kind = measured_peaks()
    ms_step = res["ms_total"] / args.steps
    value = whole_job_gbps(res["bytes_step"], ms_step, world)
    achieved_per_gpu = res["bytes_step"] / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "l2": f"inputs larger than L2: {res['R']} rotating weight copies of "
                         f"{res['per_copy_bytes'] / 2**20:.1f} MiB",
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "timing": "CUDA graph per step, CUDA events on the launching stream; "
                             "per call: graphs of 200 calls over the weight ring, median of 5 "
                             "replays",
                   "pdl": args.pdl},
        "per_call": res["per_case"],
        "gpu_launches": res["launches_per_step"] * args.steps,
        "clocks": res["clocks"],
    }
    # the roofline of the dominant kernel of the step (the most time per
    # step): algorithmic bytes of its calls / their measured time; the step
    # aggregate beside it
    by_kernel = {}
    for c in res["per_case"]:
        name = "+".join(KERNEL_OF_ROUTE[k] for k in c["kernels"])
        k = by_kernel.setdefault(name, {"us": 0.0, "bytes": 0, "launches": 0})
        k["us"] += c["us"]
        k["bytes"] += c["bytes"]
        k["launches"] += len(c["kernels"])
    for name, k in by_kernel.items():
        gbps = k["bytes"] / k["us"] / 1e3
        by_kernel[name] = {"us_per_step": round(k["us"], 2), "GBps": round(gbps, 1),
                           "frac": round(gbps / peak, 4),
                           "algorithmic_bytes_per_launch": round(k["bytes"] / k["launches"])}
    dom = max(by_kernel, key=lambda n: by_kernel[n]["us_per_step"])
    line["roofline"] = {"bound": "hbm", "achieved": by_kernel[dom]["GBps"], "peak": peak,
                        "unit": "GB/s", "frac": by_kernel[dom]["frac"], "peak_kind": peak_kind,
                        "traffic": None, "kernel": dom,
                        "step_aggregate": {"achieved": round(achieved_per_gpu, 1),
                                           "frac": round(achieved_per_gpu / peak, 4)},
                        "by_kernel": by_kernel}
    tr = recorded_traffic()
    if tr is not None and dom in tr.get("kernels", {}):
        t = tr["kernels"][dom]
        line["roofline"]["traffic"] = round(t["dram_bytes_per_launch"])
        line["roofline"]["traffic_per"] = "launch (mean over the step's launches of it, ncu)"
        line["roofline"]["traffic_source"] = tr["source"]
    if res.get("shapes"):
        for label, e in res["shapes"].items():
            for key, v in e.items():
                if isinstance(v, dict) and "GBps" in v:
                    v["frac"] = round(v["GBps"] / peak, 4)
        line["shapes"] = res["shapes"]
    if res.get("isolated"):
        for key, v in res["isolated"].items():
            if isinstance(v, dict):
                v["frac"] = round(v["GBps"] / peak, 4)
        line["isolated_m1"] = res["isolated"]
    if res.get("stacked"):
        line["stacked_gate_up"] = res["stacked"]
    if res.get("per_precision_offsets"):
        line["per_precision_offsets"] = res["per_precision_offsets"]
    m1 = [c for c in res["per_case"] if c["M"] == 1]
    line["headline_m1"] = {f"p{c['p']}": {"us": c["us"], "GBps": c["GBps"],
                                          "frac": round(c["GBps"] / peak, 4)} for c in m1}
    if "e2e" in res:
        e = res["e2e"]
        line["e2e"] = {"value": round(whole_job_gbps(res["bytes_step"], e["ms"] / e["steps"], world), 2),
                       "unit": "GB/s", "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                       "ms_per_step": round(e["ms"] / e["steps"], 4),
                       "path": "bcq_gemm_host (pinned host x/y, copies on the call's stream); "
                               "calls alternate between two streams, each with its own "
                               "staging buffers and workspace"}
    if quant is not None:
        line["quantizer"] = quant
    if rank == 0 and world == 1 and not args.profile:
        if quant is not None:
            quant["cpu_oracle"] = run_quantizer_oracle(args.seed)
        secs, by, thr = 0.0, 0.0, 1
        for k in range(max(1, args.cpu_reps)):
            s_k, b_k, thr = run_oracle_sample(args.seed + k, args.cpu_rows)
            secs += s_k
            by += b_k
        line["cpu_baseline"] = {"value": round(by / secs / 1e9, 4), "unit": "GB/s", "cores": thr,
                                "kind": "oracle",
                                "sample": f"{args.cpu_rows} of {N_OUT} output rows of each of the "
                                          f"15 calls, {max(1, args.cpu_reps)} times ({secs:.1f} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
