#!/usr/bin/env python
"""Benchmark of the NVFP4 linear path on B200: prints ONE JSON line (rank 0).

Step = one forward pass of a stack of L distinct DiT layers at M = 41 tokens, hidden 1536
(per layer: AdaLN->FP4, QKV GEMM +bias, context quantize, attention-output GEMM
+bias+residual, LayerNorm->FP4, FFN-up GEMM +bias+tanh-GELU->FP4, FFN-down GEMM
+bias+residual: 7 kernels), replayed from a CUDA graph.  L = 24 puts 382 MB of distinct
weights behind each step, 3x the 126 MB L2, so every layer streams its weights from HBM.
Metric: microseconds per layer (lower is better), plus the weight-stream GB/s it implies.

Side measurements in the same line: the GEMM kernel's roofline (CUDA events around graph
replays of each DiT GEMM over L distinct weight copies), the M = 968 prefill layer's
TFLOPS (tensor-bound), the 18-layer action-expert stack, the M sweep on 1536 -> 6144, and
the oracle on the host cores (cpu_baseline).

--impl reference times the oracle (the benchmark's reference arm) on the same workload.
Multi-GPU (torchrun): independent replicas, one per rank; timing is the max over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 linear µs/layer & weight-stream GB/s at M=41; TFLOPS at M=968"
UNIT = "µs/layer"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0  # nominal dense ratio, 9 PF / 2.25 PF
DIT = dict(M=41, H=1536, F=6144)

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernels,
# from one ncu capture of each kernel (`ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum
# --clock-control none -k regex:<kernel>` over `bench.py --profile-case <case>`), keyed by a hash
# of the kernel sources they were taken on: once a source changes the figure is reported as null.
TRAFFIC = {
    "dit_gemm": {"sources": ["gemm.cu", "gemm.h", "epilogue.cuh", "quant.cuh", "sm100.cuh"],
                 "sha256": "e533d6ba7a6374968bbe10c65e2504292a354537b26dbd3bd82c9cbf495935a7",
                 "bytes": 4214336},  # mean of the 4 DiT GEMM launches (case dit-gemms)
    "prefill_gate_up": {"sources": ["gemm_persistent.cu", "gemm.h", "epilogue.cuh", "quant.cuh", "sm100.cuh"],
                        "sha256": "31ab8efdad49dbafc019494c7a579955034a47b345434bb78976656d20918f52",
                        "bytes": 38947072},  # the gate/up launch of case prefill-gemms
}


def sources_sha(names):
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "vla_action_head_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic(key):
    t = TRAFFIC[key]
    if t["bytes"] is None or t["sha256"] != sources_sha(t["sources"]):
        return None
    return t["bytes"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=24)
    ap.add_argument("--no-side", action="store_true", help="skip the side measurements")
    ap.add_argument("--soak-steps", type=int, default=200,
                    help="untimed steps while the clock sampler starts (0 for profiling runs)")
    ap.add_argument("--profile-case", default=None,
                    help="run one small case for ncu (dit-gemms | prefill-gemms | grouped | norm) or the traced "
                         "DiT launch chain (dit-chain-trace), and exit")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


class Clocks:
    """nvidia-smi sampler (every 100 ms) bracketing a timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, v, device="cuda"):
    """The largest v over the ranks (every rank gets it); `device` is where the collective
    runs ("cuda" under NCCL, "cpu" under gloo)."""
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def us_per_layer(ms_max, steps, layers_per_step, ws):
    """Whole-job time per layer: every rank runs `steps` x `layers_per_step` layers of its own
    (replicas), the job ends with the slowest rank."""
    return ms_max * 1e3 / (steps * layers_per_step * ws)


# ---------------------------------------------------------------------------------------
def gemm_bytes(M, N, K, epi):
    """Algorithmic bytes of one GEMM: A and W codes + scales, output, bias, residual."""
    b = M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16
    if epi == "geglu":
        b += M * (N // 2) // 2 + M * (N // 2) // 16
    elif epi == "bias_gelu":
        b += M * N // 2 + M * N // 16
    else:
        b += 2 * M * N
    if epi in ("bias", "bias_residual", "bias_gelu"):
        b += 2 * N
    if epi in ("residual", "bias_residual"):
        b += 2 * M * N
    return b


SOAK_S = 0.3  # untimed replays before a side measurement, so its clock sampler sees the load


def time_graph(g, reps, stream, soak_s=None):
    """ms per replay; replays and events on `stream`.  Before the timed replays the graph
    replays untimed for about soak_s seconds (SOAK_S by default)."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    soak_s = SOAK_S if soak_s is None else soak_s
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        t_end = time.perf_counter() + soak_s
        while time.perf_counter() < t_end:
            for _ in range(8):
                g.replay()
            torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def capture(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def gemm_ring_time(A, lins, epi, outs, ws, stream, reps=20, res=None):
    """Average time (ms) of one GEMM launch over a graph of len(lins) distinct weights."""
    from vla_action_head_b200 import nvfp4

    def body():
        for i, lin in enumerate(lins):
            nvfp4.gemm(A, lin.w, epi, bias=lin.bias, residual=res, out=outs[i % len(outs)], workspace=ws)
    body()  # sizes the workspace before capture
    g = capture(body, stream)
    ms = time_graph(g, reps, stream)
    del g
    return ms / len(lins)


# ---------------------------------------------------------------------------------------
def cpu_baseline_dit(steps=1, threads=1):
    """The oracle (single-threaded C, fp64 GEMM) on one full DiT layer at M = 41.  threads > 1:
    the GEMMs' output rows are partitioned over that many host threads (the oracle call
    releases the interpreter lock), the norms stay on one thread."""
    import numpy as np
    import torch

    from oracle import oracle as orc
    from vla_action_head_b200 import synth

    M, H, F = DIT["M"], DIT["H"], DIT["F"]
    s = lambda tid: synth.seed_of(2, tid)  # noqa: E731
    cpu = lambda seed, shape, m, sd: synth.bf16_normal_torch(seed, shape, m, sd, device="cpu").view(  # noqa: E731
        torch.int16).numpy().view(np.uint16)
    x = cpu(s(synth.X), (M, H), 0, 1)
    ctx = cpu(s(synth.CONTEXT), (M, H), 0, 1)
    sc, sh = cpu(s(synth.MOD_SCALE), (H,), 0, 0.1), cpu(s(synth.MOD_SHIFT), (H,), 0, 0.1)
    ga, be = cpu(s(synth.GAMMA), (H,), 1, 0.1), cpu(s(synth.BETA), (H,), 0, 0.1)
    shapes = [(3 * H, H), (H, H), (F, H), (H, F)]
    W = [orc.quantize_weight(cpu(s(synth.W0 + i), shp, 0, 0.02)) for i, shp in enumerate(shapes)]
    B = [cpu(s(synth.BIAS0 + i), (shp[0],), 0, 0.01) for i, shp in enumerate(shapes)]

    def bf16(v):
        return synth.f32_to_bf16_bits(v.astype(np.float32))

    pool = None
    if threads > 1:
        from concurrent.futures import ThreadPoolExecutor
        pool = ThreadPoolExecutor(threads)

    def gemm(*a, **kw):
        if pool is None:
            return orc.gemm(*a, **kw)
        parts = np.array_split(np.arange(M), threads)
        res = list(pool.map(lambda r: orc.gemm(*a, rows=r, **kw), parts))
        out = {"v": np.concatenate([r["v"] for r in res])}
        if res[0]["codes"] is not None:  # each part fills its own rows of zeroed buffers
            out["codes"] = np.bitwise_or.reduce([r["codes"] for r in res])
            out["sf"] = np.bitwise_or.reduce([r["sf"] for r in res])
        return out

    t0 = time.perf_counter()
    for _ in range(steps):
        a1, a1s = orc.quantize_norm(x, "adaln", scale=sc, shift=sh, eps=1e-6)
        gemm(a1, a1s, 1.0, M, W[0][0], W[0][1], W[0][2], 3 * H, H, epi="bias", bias=B[0])
        c, cs = orc.quantize_norm(ctx, "none")
        h = bf16(gemm(c, cs, 1.0, M, W[1][0], W[1][1], W[1][2], H, H, epi="bias_residual", bias=B[1],
                      residual=x)["v"])
        a2, a2s = orc.quantize_norm(h, "layernorm", gamma=ga, beta=be, eps=1e-5)
        u = gemm(a2, a2s, 1.0, M, W[2][0], W[2][1], W[2][2], F, H, epi="bias_gelu", bias=B[2])
        gemm(u["codes"], u["sf"], 1.0, M, W[3][0], W[3][1], W[3][2], H, F, epi="bias_residual",
             bias=B[3], residual=h)
    dt = time.perf_counter() - t0
    if pool is not None:
        pool.shutdown()
    return dt / steps * 1e6  # us per layer


def _cpu_bits(seed, shape, mean, std):
    import numpy as np
    import torch

    from vla_action_head_b200 import synth
    return synth.bf16_normal_torch(seed, shape, mean, std, device="cpu").view(torch.int16).numpy().view(np.uint16)


def _rows_gemm(threads):
    """orc.gemm, with the output rows split over `threads` host threads when > 1 (the oracle
    call releases the interpreter lock)."""
    import numpy as np

    from oracle import oracle as orc
    if threads <= 1:
        return orc.gemm, None
    from concurrent.futures import ThreadPoolExecutor
    pool = ThreadPoolExecutor(threads)

    def gemm(*a, rows=None, **kw):
        M = a[3]
        sel = np.arange(M) if rows is None else np.asarray(rows)
        parts = [p for p in np.array_split(sel, threads) if len(p)]
        res = list(pool.map(lambda r: orc.gemm(*a, rows=r, **kw), parts))
        out = {"v": np.concatenate([r["v"] for r in res])}
        if res[0]["codes"] is not None:  # each part fills its own rows of zeroed buffers
            out["codes"] = np.bitwise_or.reduce([r["codes"] for r in res])
            out["sf"] = np.bitwise_or.reduce([r["sf"] for r in res])
        return out
    return gemm, pool


def cpu_baseline_tiny(reps=3, threads=1):
    """The oracle on the tiny workload: LayerNorm -> NVFP4 of 41 x 256, GEMM 41 x 512 x 256 +
    bias.  us per norm + GEMM (mean of `reps`)."""
    from oracle import oracle as orc
    from vla_action_head_b200 import synth
    s = lambda tid: synth.seed_of(1, tid)  # noqa: E731
    x = _cpu_bits(s(synth.X), (41, 256), 0, 1)
    ga, be = _cpu_bits(s(synth.GAMMA), (256,), 1, 0.1), _cpu_bits(s(synth.BETA), (256,), 0, 0.1)
    wc, wsf, gw = orc.quantize_weight(_cpu_bits(s(synth.W0), (512, 256), 0, 0.02))
    bias = _cpu_bits(s(synth.BIAS0), (512,), 0, 0.01)
    gemm, pool = _rows_gemm(threads)
    t0 = time.perf_counter()
    for _ in range(reps):
        a, asf = orc.quantize_norm(x, "layernorm", gamma=ga, beta=be, eps=1e-5)
        gemm(a, asf, 1.0, 41, wc, wsf, gw, 512, 256, epi="bias", bias=bias)
    dt = (time.perf_counter() - t0) / reps
    if pool is not None:
        pool.shutdown()
    return dt * 1e6


def cpu_baseline_ae(reps=3, threads=1):
    """The oracle on one action-expert layer (M = 50, width 1024, context 2048, gated MLP
    2 x 4096): 2 AdaRMSNorm -> NVFP4, context quantize, QKV, o + residual, gate/up GeGLU ->
    FP4, down + residual.  us per layer (mean of `reps`)."""
    from oracle import oracle as orc
    from vla_action_head_b200 import synth
    s = lambda tid: synth.seed_of(3, tid)  # noqa: E731
    M, H, A, F = 50, 1024, 2048, 4096
    x = _cpu_bits(s(synth.X), (M, H), 0, 1)
    ctx = _cpu_bits(s(synth.CONTEXT), (M, A), 0, 1)
    s1, s2 = _cpu_bits(s(synth.MOD_SCALE), (H,), 0, 0.1), _cpu_bits(s(synth.MOD_SHIFT), (H,), 0, 0.1)
    shapes = [(2560, H), (H, A), (2 * F, H), (H, F)]
    W = [orc.quantize_weight(_cpu_bits(s(synth.W0 + i), shp, 0, 0.02), interleave_gate_up=(i == 2))
         for i, shp in enumerate(shapes)]
    gemm, pool = _rows_gemm(threads)
    t0 = time.perf_counter()
    for _ in range(reps):
        a1, a1s = orc.quantize_norm(x, "adarms", scale=s1, eps=1e-6)
        gemm(a1, a1s, 1.0, M, *W[0], 2560, H, epi="none")
        c, cs = orc.quantize_norm(ctx, "none")
        h = synth.f32_to_bf16_bits(gemm(c, cs, 1.0, M, *W[1], H, A, epi="residual", residual=x)["v"])
        a2, a2s = orc.quantize_norm(h, "adarms", scale=s2, eps=1e-6)
        u = gemm(a2, a2s, 1.0, M, *W[2], 2 * F, H, epi="geglu")
        gemm(u["codes"], u["sf"], 1.0, M, *W[3], H, F, epi="residual", residual=h)
    dt = (time.perf_counter() - t0) / reps
    if pool is not None:
        pool.shutdown()
    return dt * 1e6


def _fit_rows(run, M, threads, per_thread=(8, 24)):
    """Time run(rows) on two evenly spread row samples of per_thread x threads rows each (best
    of two), fit t = a + b x rows (a: the weight decode each call repeats, b: the products of
    one row) and evaluate at M rows.  Returns (us, the sample sizes)."""
    import numpy as np
    ns = [min(M, k * threads) for k in per_thread]
    ts = []
    for n in ns:
        sel = np.linspace(0, M - 1, n).astype(np.int64)
        best = None
        for _ in range(2):
            t0 = time.perf_counter()
            run(sel)
            dt = time.perf_counter() - t0
            best = dt if best is None else min(best, dt)
        ts.append(best)
    if ns[1] == ns[0]:
        return ts[0] * 1e6, ns
    slope = (ts[1] - ts[0]) / (ns[1] - ns[0])
    return (ts[0] + slope * (M - ns[0])) * 1e6, ns


def cpu_baseline_prefill(threads=1):
    """The oracle on one prefill layer (M = 968, width 2048, MLP 2 x 16384): 2 RMSNorm ->
    NVFP4 over all rows, and the three GEMMs timed on two row samples and extrapolated in
    rows (_fit_rows).  Returns (us per layer, description of the sample)."""
    from oracle import oracle as orc
    from vla_action_head_b200 import synth
    s = lambda tid: synth.seed_of(4, tid)  # noqa: E731
    M, H, F = 968, 2048, 16384
    x = _cpu_bits(s(synth.X), (M, H), 0, 1)
    g1, g2 = _cpu_bits(s(synth.GAMMA), (H,), 1, 0.1), _cpu_bits(s(synth.BETA), (H,), 1, 0.1)
    Wq = orc.quantize_weight(_cpu_bits(s(synth.W0), (2560, H), 0, 0.02))
    Wg = orc.quantize_weight(_cpu_bits(s(synth.W0 + 2), (2 * F, H), 0, 0.02), interleave_gate_up=True)
    Wd = orc.quantize_weight(_cpu_bits(s(synth.W0 + 3), (H, F), 0, 0.02))
    gemm, pool = _rows_gemm(threads)
    t0 = time.perf_counter()
    a1, a1s = orc.quantize_norm(x, "rmsnorm", gamma=g1, eps=1e-6)
    a2, a2s = orc.quantize_norm(x, "rmsnorm", gamma=g2, eps=1e-6)
    t_norm = time.perf_counter() - t0

    def gemms(sel):
        gemm(a1, a1s, 1.0, M, *Wq, 2560, H, epi="none", rows=sel)
        u = gemm(a2, a2s, 1.0, M, *Wg, 2 * F, H, epi="geglu", rows=sel)
        # u holds the sampled rows (the rest zero): the down GEMM reads the same rows
        gemm(u["codes"], u["sf"], 1.0, M, *Wd, H, F, epi="residual", residual=x, rows=sel)
    us, ns = _fit_rows(gemms, M, threads)
    if pool is not None:
        pool.shutdown()
    return t_norm * 1e6 + us, (f"norms over all 968 rows; the 3 GEMMs timed on {ns[0]} and {ns[1]} sampled rows "
                               "and extrapolated linearly in rows to 968")


def cpu_baseline_sweep(threads=1):
    """The oracle on the 1536 -> 6144 GEMM (+bias) at each M of the sweep; M > 41 timed on
    two row samples and extrapolated in rows (_fit_rows).  {M: us}."""
    from oracle import oracle as orc
    from vla_action_head_b200 import synth
    W = orc.quantize_weight(_cpu_bits(synth.seed_of(5, 1000), (6144, 1536), 0, 0.02))
    bias = _cpu_bits(synth.seed_of(5, 2000), (6144,), 0, 0.01)
    gemm, pool = _rows_gemm(threads)
    out = {}
    for Ms in (1, 16, 41, 128, 512, 968):
        a, asf = orc.quantize_norm(_cpu_bits(synth.seed_of(5, Ms), (Ms, 1536), 0, 1), "none")
        if Ms <= 41:
            t0 = time.perf_counter()
            gemm(a, asf, 1.0, Ms, *W, 6144, 1536, epi="bias", bias=bias)
            out[Ms] = (time.perf_counter() - t0) * 1e6
            continue
        out[Ms], _ = _fit_rows(lambda sel: gemm(a, asf, 1.0, Ms, *W, 6144, 1536, epi="bias", bias=bias, rows=sel),
                               Ms, threads)
    if pool is not None:
        pool.shutdown()
    return out


def cpu_baselines_all(nthr):
    """The oracle beside every workload, single-threaded and on `nthr` host threads."""
    res = {}
    for name, fn, unit, reps in [("tiny_41x256_512", cpu_baseline_tiny, "µs per norm + GEMM", 3),
                                 ("action_expert_layer_m50", cpu_baseline_ae, "µs/layer", 3)]:
        for thr in (1, nthr):
            us = fn(reps=reps, threads=thr)
            res.setdefault(name, {"unit": unit, "kind": "oracle", "sample": f"the whole workload, mean of {reps}"})
            res[name]["us_1_thread" if thr == 1 else f"us_{nthr}_threads"] = round(us, 1)
    for thr in (1, nthr):
        us, sample = cpu_baseline_prefill(threads=thr)
        res.setdefault("prefill_layer_m968", {"unit": "µs/layer", "kind": "oracle", "sample": sample})
        res["prefill_layer_m968"]["us_1_thread" if thr == 1 else f"us_{nthr}_threads"] = round(us, 1)
    for thr in (1, nthr):
        sw = cpu_baseline_sweep(threads=thr)
        res.setdefault("m_sweep_1536x6144", {"unit": "µs per GEMM", "kind": "oracle",
                                             "sample": "M <= 41 whole; larger M on 8 and 24 sampled rows per "
                                                       "thread, extrapolated linearly in rows"})
        res["m_sweep_1536x6144"]["us_1_thread" if thr == 1 else f"us_{nthr}_threads"] = {
            str(k): round(v, 1) for k, v in sw.items()}
    return res


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def reference_arm(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # each step is one full DiT layer on the oracle (~1.6 s); the run is bounded to ~3 min by
    # timing at most as many of the K steps as fit, which the line states in its sample
    t0 = time.perf_counter()
    cpu_baseline_dit(1)
    per = time.perf_counter() - t0
    for _ in range(max(0, min(args.warmup, int(30 / per)) - 1)):
        cpu_baseline_dit(1)
    n = max(1, min(args.steps, int(150 / max(per, 1e-3))))
    us = cpu_baseline_dit(n)
    line = {"metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "one DiT layer, M=41, hidden 1536, FFN 6144 (oracle, fp64 GEMM)",
                       "global_batch": DIT["M"], "parallelism": "replicas" if ws > 1 else "single"},
            "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"one full DiT layer per step; {n} of {args.steps} steps timed"},
            "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
def profile_case(name):
    """Small, short runs of single kernels for ncu (a few launches, a few hundred MB)."""
    import torch

    from vla_action_head_b200 import layers, nvfp4
    torch.cuda.set_device(0)
    nvfp4.probe()
    if name == "dit-gemms":
        lay = layers.DiTLayer(**DIT)
        x = torch.randn(DIT["M"], DIT["H"], device="cuda").to(torch.bfloat16)
        y = torch.empty_like(x)
        for _ in range(3):
            lay.forward(x, x, y)
    elif name == "prefill-gemms":
        lay = layers.PrefillLayer()
        x = torch.randn(968, 2048, device="cuda").to(torch.bfloat16)
        y = torch.empty_like(x)
        for _ in range(3):
            lay.forward(x, x, y)
    elif name == "grouped":
        M, H, G = DIT["M"], DIT["H"], 32
        ctxq = nvfp4.quantize_norm(torch.randn(M, H, device="cuda").to(torch.bfloat16), "none")
        outs = [torch.empty((M, H), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        lins = [layers.Linear(0.02 * torch.randn(H, H, device="cuda").to(torch.bfloat16)) for _ in range(G)]
        grp = nvfp4.GroupedGemm([(ctxq, l.w, outs[g]) for g, l in enumerate(lins)])
        for _ in range(3):
            grp.run()
    elif name == "dit-chain-trace":
        # per-CTA timestamps of the launch chain: a CUDA graph of 8 DiT layers (distinct weights)
        # with nvfp4_set_gemm_trace; prints, per GEMM launch, the medians over its CTAs of the
        # stamps and the gap from the previous launch's last exit to this one's first stage
        import numpy as np

        from vla_action_head_b200 import synth
        L = nvfp4.lib()
        R, (M, H, F) = 8, (DIT["M"], DIT["H"], DIT["F"])
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            wsp = nvfp4.Workspace("cuda")
            lays = [layers.DiTLayer(**DIT, layer=i, ws=wsp) for i in range(R)]
            x0 = synth.bf16_normal_torch(synth.seed_of(2, synth.X), (M, H), device="cuda")
            ctx = synth.bf16_normal_torch(synth.seed_of(2, synth.CONTEXT), (M, H), device="cuda")
            buf = [x0.clone(), torch.empty_like(x0)]

            def fwd():
                for i, lay in enumerate(lays):
                    lay.forward(buf[i % 2], ctx, buf[(i + 1) % 2])
            fwd()
        torch.cuda.synchronize()
        gemms = [("qkv", 3 * H, H, "bias"), ("o", H, H, "bias_residual"), ("up", F, H, "bias_gelu"),
                 ("down", H, F, "bias_residual")]
        words = [int(L.nvfp4_gemm_trace_words(M, N, K, nvfp4.EPI[e])) for _, N, K, e in gemms]
        tr = torch.zeros(sum(words) * R, dtype=torch.int64, device="cuda")
        L.nvfp4_set_gemm_trace(tr.data_ptr(), tr.numel())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fwd()
        L.nvfp4_set_gemm_trace(None, 0)
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        tr.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        t = tr.cpu().numpy().astype(np.float64)
        t0 = t[t > 0].min()
        off, prev_exit = 0, None
        labels = [(0, "entry"), (3, "first stage"), (4, "last MMA"), (5, "acc ready"), (7, "partials in"),
                  (1, "epilogue done"), (6, "exit")]
        print("per launch, us from the first stamp (median over CTAs / max)")
        for k in range(4 * R):
            n = words[k % 4]
            blk = t[off:off + n].reshape(-1, 8)
            off += n
            rel = (blk - t0) / 1e3
            cols = []
            for c, lab in labels:
                v = rel[:, c][blk[:, c] > 0]
                if len(v):
                    cols.append(f"{lab} {np.median(v):7.2f}/{v.max():7.2f}")
            first = rel[:, 3][blk[:, 3] > 0]
            gap = "" if prev_exit is None else f" | gap {np.median(first) - prev_exit:5.2f}"
            prev_exit = rel[:, 6][blk[:, 6] > 0].max()
            print(f"{gemms[k % 4][0]:5s} L{k // 4} ({n // 8} CTAs) " + " | ".join(cols) + gap)
        del g
    elif name == "norm":
        x = torch.randn(968, 2048, device="cuda").to(torch.bfloat16)
        g = torch.ones(2048, device="cuda").to(torch.bfloat16)
        for _ in range(3):
            nvfp4.quantize_norm(x, "rmsnorm", gamma=g)
    torch.cuda.synchronize()
    nvfp4.device_status()
    print(json.dumps({"profile_case": name, "ok": True}))


def main():
    args = parse()
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile_case:
        return profile_case(args.profile_case)
    import torch

    from vla_action_head_b200 import build, layers, nvfp4, synth
    build.build()
    ws_n, rank, local = dist_setup()
    nvfp4.probe()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream()
    pk, pk_kind = peaks()
    L, M, H, F = args.layers, DIT["M"], DIT["H"], DIT["F"]

    # ---- the DiT stack (main metric) ----
    with torch.cuda.stream(stream):
        wsp = nvfp4.Workspace(dev)
        stack = [layers.DiTLayer(**DIT, layer=i, device=dev, ws=wsp) for i in range(L)]
        x0 = synth.bf16_normal_torch(synth.seed_of(2, synth.X), (M, H), device=dev)
        ctx = synth.bf16_normal_torch(synth.seed_of(2, synth.CONTEXT), (M, H), device=dev)
        buf = [x0.clone(), torch.empty_like(x0)]
    torch.cuda.synchronize()

    def stack_fwd():
        for i, lay in enumerate(stack):
            lay.forward(buf[i % 2], ctx, buf[(i + 1) % 2])

    with torch.cuda.stream(stream):
        stack_fwd()  # eager pass: sizes the workspace, loads the kernels
    torch.cuda.synchronize()
    nvfp4.device_status()
    g_stack = capture(stack_fwd, stream)

    def run_steps(n, with_copies=None):
        for _ in range(n):
            if with_copies:
                buf[0].copy_(with_copies[0], non_blocking=True)
            g_stack.replay()
            if with_copies:
                with_copies[1].copy_(buf[L % 2], non_blocking=True)

    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    torch.cuda.synchronize()
    barrier(ws_n)
    clk = Clocks(local)
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        run_steps(args.soak_steps)  # so the clock sampler sees the load
    torch.cuda.synchronize()
    barrier(ws_n)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        run_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws_n)
    clocks = clk.stop()
    ms_total = max_over_ranks(ws_n, e0.elapsed_time(e1))
    nvfp4.device_status()
    us_layer = us_per_layer(ms_total, args.steps, L, ws_n)
    # per-step spread (each step timed on its own, after the timed region)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with torch.cuda.stream(stream):
        evs[0].record(stream)
        for i in range(args.steps):
            run_steps(1)
            evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per_step = sorted(evs[i].elapsed_time(evs[i + 1]) * 1e3 / L for i in range(args.steps))
    spread = {"median": round(statistics.median(per_step), 3),
              "p95": round(per_step[min(len(per_step) - 1, int(0.95 * len(per_step)))], 3),
              "unit": UNIT, "steps": args.steps}
    w_bytes = sum(l.weight_bytes() for l in stack[0].linears())
    gbs_weights = w_bytes / (us_layer * 1e-6) / 1e9

    # ---- end to end through the same API with host buffers ----
    xh = torch.empty((M, H), dtype=torch.bfloat16).pin_memory()
    yh = torch.empty((M, H), dtype=torch.bfloat16).pin_memory()
    xh.copy_(x0.cpu())
    with torch.cuda.stream(stream):
        run_steps(2, (xh, yh))
    torch.cuda.synchronize()
    barrier(ws_n)
    e0.record(stream)
    with torch.cuda.stream(stream):
        run_steps(args.steps, (xh, yh))
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws_n)
    ms_e2e = max_over_ranks(ws_n, e0.elapsed_time(e1))
    us_layer_e2e = us_per_layer(ms_e2e, args.steps, L, ws_n)

    line = {"metric": METRIC, "value": round(us_layer, 3), "unit": UNIT, "n_gpus": ws_n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_total / args.steps, 4), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x ue4m3) -> fp32 acc; bf16 io",
            "data": "synthetic",
            "config": {"workload": f"DiT layer stack, {L} distinct layers per step, M=41 tokens, hidden 1536, "
                                   "FFN 6144, AdaLN/LayerNorm->NVFP4, 4 NVFP4 GEMMs with fused epilogues",
                       "global_batch": M, "layers_per_step": L, "parallelism": f"replicas x{ws_n}",
                       "l2": f"inputs larger than L2: {L} x {w_bytes / 1e6:.1f} MB distinct weights per step",
                       "graph": "CUDA graph replay, programmatic dependent launch"},
            "weight_stream_gbs": round(gbs_weights, 1),
            "per_step_us_per_layer": spread,
            "clocks": clocks,
            "gpu_launches": args.steps * L * layers.DiTLayer.launches,
            "e2e": {"value": round(us_layer_e2e, 3), "unit": UNIT, "h2d_bytes_per_step": M * H * 2,
                    "d2h_bytes_per_step": M * H * 2}}

    del g_stack
    if not args.no_side:
        try:
            line.update(side_measurements(stack, wsp, stream, dev, pk, pk_kind))
        except Exception as e:  # a side measurement never hides the main line
            line["side_error"] = repr(e)[:300]
    if rank == 0 and ws_n == 1 and not args.no_side:
        try:
            us_cpu = cpu_baseline_dit(1)
            line["cpu_baseline"] = {"value": round(us_cpu, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
                                    "sample": "one full DiT layer (M=41, hidden 1536, FFN 6144), fp64 GEMM, "
                                              "single-threaded C", "cpu_model": cpu_model()}
        except Exception as e:  # the baseline is reported, never required
            line["cpu_baseline"] = {"value": None, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": str(e)}
        try:
            nthr = len(os.sched_getaffinity(0))
            us_mt = cpu_baseline_dit(1, threads=nthr)
            line["cpu_baseline_threads"] = {"value": round(us_mt, 1), "unit": UNIT, "cores": nthr,
                                            "kind": "oracle", "sample": "the same DiT layer, GEMM output rows "
                                            f"partitioned over {nthr} host threads"}
        except Exception as e:
            line["cpu_baseline_threads"] = {"value": None, "sample": str(e)[:200]}
        try:
            line["cpu_baseline_configs"] = cpu_baselines_all(len(os.sched_getaffinity(0)))
        except Exception as e:
            line["cpu_baseline_configs"] = {"error": repr(e)[:200]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


class ClockRecord:
    """Samples the GPU clocks over one side measurement and stores them in entry["clocks"]."""

    def __init__(self, gpu_index, entry_of):
        self.gpu, self.entry_of = gpu_index, entry_of

    def __enter__(self):
        self.clk = Clocks(self.gpu)
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        rec = self.clk.stop()
        if exc[0] is None:
            self.entry_of()["clocks"] = rec
        return False


def side_measurements(stack, wsp, stream, dev, pk, pk_kind):
    import torch

    from vla_action_head_b200 import layers, nvfp4, synth
    M, H, F = DIT["M"], DIT["H"], DIT["F"]
    out = {}
    gpu = dev.index if dev.index is not None else 0
    fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16

    def clocked(key):
        return ClockRecord(gpu, lambda: out[key])

    # ---- roofline of the GEMM kernel in the DiT layer (HBM-bound at M = 41) ----
    l0 = stack[0]
    per = {}
    tot_b, tot_ms = 0, 0.0
    specs = [("qkv", l0.a1, "qkv", "bias", 3 * H, H), ("attn_out", l0.ctx_q, "o", "bias_residual", H, H),
             ("ffn_up", l0.a2, "up", "bias_gelu", F, H), ("ffn_down", l0.u, "down", "bias_residual", H, F)]
    res = torch.zeros((M, H), dtype=torch.bfloat16, device=dev)
    with clocked("roofline"):
        with torch.cuda.stream(stream):
            for name, A, attr, epi, N, K in specs:
                lins = [getattr(s, attr) for s in stack]
                if epi == "bias_gelu":
                    outs = [nvfp4.empty_fp4(M, N, dev) for _ in range(2)]
                else:
                    outs = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
                ms = gemm_ring_time(A, lins, epi, outs, wsp, stream, res=res if "residual" in epi else None)
                b = gemm_bytes(M, N, K, epi)
                per[name] = {"us": round(ms * 1e3, 3), "gbs": round(b / (ms * 1e-3) / 1e9, 1), "bytes": b}
                tot_b += b
                tot_ms += ms
        ach = tot_b / (tot_ms * 1e-3) / 1e9
        out["roofline"] = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": round(ach / pk["hbm_gbs"], 4), "traffic": traffic("dit_gemm"),
                           "algorithmic_bytes_per_launch": tot_b // len(specs),
                           "kernel": "gemm_kernel (4 DiT GEMMs, M=41, L2-cold weights)", "peak_kind": pk_kind,
                           "per_gemm": per}
    # ---- grouped GEMM: 32 cross-attention K/V projections of one M = 41 context in one
    # launch; a ring of 4 groups with distinct weights (4 x 42.5 MB > L2) ----
    with torch.cuda.stream(stream):
        Kc, Nc, G = H, H, 32
        ctxq = nvfp4.quantize_norm(synth.bf16_normal_torch(synth.seed_of(7, synth.CONTEXT), (M, Kc), device=dev),
                                   "none")
        groups, kv_outs = [], [torch.empty((M, Nc), dtype=torch.bfloat16, device=dev) for _ in range(G)]
        kv_lins = []
        for r in range(4):
            ls = [layers.Linear(synth.bf16_normal_torch(synth.seed_of(7, 3000 + 64 * r + g), (Nc, Kc), 0, 0.02,
                                                        device=dev)) for g in range(G)]
            kv_lins.append(ls)
            groups.append(nvfp4.GroupedGemm([(ctxq, l.w, kv_outs[g]) for g, l in enumerate(ls)]))

        def grouped():
            for grp in groups:
                grp.run()

        def chained():
            for ls in kv_lins:
                for g, l in enumerate(ls):
                    nvfp4.gemm(ctxq, l.w, "none", out=kv_outs[g], workspace=wsp)
        grouped()
        chained()
    torch.cuda.synchronize()
    with clocked("grouped_cross_kv32"):
        g = capture(grouped, stream)
        ms_g = time_graph(g, 20, stream) / len(groups)
        del g
        g = capture(chained, stream)
        ms_c = time_graph(g, 20, stream) / len(groups)
        del g
        b_grp = G * gemm_bytes(M, Nc, Kc, "none")
        out["grouped_cross_kv32"] = {"problems": f"{G} x {M}x{Nc}x{Kc}, shared context",
                                     "us": round(ms_g * 1e3, 2), "gbs": round(b_grp / (ms_g * 1e-3) / 1e9, 1),
                                     "frac_hbm": round(b_grp / (ms_g * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                                     "us_as_32_launches": round(ms_c * 1e3, 2), "bytes": b_grp,
                                     "l2": "ring of 4 groups with distinct weights (170 MB > L2)"}
    del groups, kv_lins, kv_outs, ctxq
    # ---- 18-layer action-expert stack (config 3 layers, one CUDA graph) ----
    with torch.cuda.stream(stream):
        ae = [layers.ActionExpertLayer(layer=i, device=dev, ws=wsp) for i in range(18)]
        xa = synth.bf16_normal_torch(synth.seed_of(3, synth.X), (50, 1024), device=dev)
        ca = synth.bf16_normal_torch(synth.seed_of(3, synth.CONTEXT), (50, 2048), device=dev)
        ab = [xa.clone(), torch.empty_like(xa)]

        def ae_fwd():
            for i, lay in enumerate(ae):
                lay.forward(ab[i % 2], ca, ab[(i + 1) % 2])
        ae_fwd()
    torch.cuda.synchronize()
    with clocked("action_expert_stack18"):
        g = capture(ae_fwd, stream)
        ms = time_graph(g, 50, stream)
        del g
        ae_w = sum(l.weight_bytes() for l in ae[0].linears())
        # its four GEMMs alone, each over the 18 layers' weights (L2-cold)
        a0 = ae[0]
        ae_per = {}
        res50 = torch.zeros((50, 1024), dtype=torch.bfloat16, device=dev)
        with torch.cuda.stream(stream):
            for name, A, attr, epi, N, K in [("qkv", a0.a1, "qkv", "none", 2560, 1024),
                                             ("o", a0.ctx_q, "o", "residual", 1024, 2048),
                                             ("gate_up", a0.a2, "gate_up", "geglu", 8192, 1024),
                                             ("down", a0.u, "down", "residual", 1024, 4096)]:
                outs = ([nvfp4.empty_fp4(50, N // 2, dev) for _ in range(2)] if epi == "geglu" else
                        [torch.empty((50, N), dtype=torch.bfloat16, device=dev) for _ in range(2)])
                ms_g = gemm_ring_time(A, [getattr(l, attr) for l in ae], epi, outs, wsp, stream,
                                      res=res50 if epi == "residual" else None)
                b = gemm_bytes(50, N, K, epi)
                ae_per[name] = {"us": round(ms_g * 1e3, 3), "gbs": round(b / (ms_g * 1e-3) / 1e9, 1), "bytes": b,
                                "frac_hbm": round(b / (ms_g * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        out["action_expert_stack18"] = {"us_per_stack": round(ms * 1e3, 2), "us_per_layer": round(ms * 1e3 / 18, 3),
                                        "weight_stream_gbs": round(18 * ae_w / (ms * 1e-3) / 1e9, 1),
                                        "per_gemm": ae_per}
    del ae, xa, ab
    # ---- the same stack with the gated residual updates fused into the norm front-ends ----
    with torch.cuda.stream(stream):
        gae = [layers.GatedActionExpertLayer(layer=i, device=dev, ws=wsp) for i in range(18)]
        r0 = synth.bf16_normal_torch(synth.seed_of(6, synth.X), (50, 1024), device=dev)
        rg = r0.clone()

        def gae_fwd():
            rg.copy_(r0)
            d, gate = None, None
            for lay in gae:
                d, gate = lay.forward(rg, d, gate, ca)
        gae_fwd()
    torch.cuda.synchronize()
    with clocked("gated_action_expert_stack18"):
        g = capture(gae_fwd, stream)
        ms = time_graph(g, 50, stream)
        del g
        gae_w = sum(l.weight_bytes() for l in gae[0].linears())
        out["gated_action_expert_stack18"] = {
            "us_per_stack": round(ms * 1e3, 2), "us_per_layer": round(ms * 1e3 / 18, 3),
            "weight_stream_gbs": round(18 * gae_w / (ms * 1e-3) / 1e9, 1),
            "front_end": "gated residual + AdaRMSNorm -> NVFP4 in one launch"}
    del gae, r0, rg, ca
    # ---- prefill layers at M = 968 (tensor-bound): the 18-layer stack in one CUDA graph
    # (1.07 GB of distinct weights), and each GEMM over the 18 layers' weights ----
    with torch.cuda.stream(stream):
        pre = [layers.PrefillLayer(layer=i, device=dev, ws=wsp) for i in range(18)]
        xp = synth.bf16_normal_torch(synth.seed_of(4, synth.X), (968, 2048), device=dev)
        pb = [xp.clone(), torch.empty_like(xp)]

        def pre_fwd():
            for i, lay in enumerate(pre):
                lay.forward(pb[i % 2], pb[i % 2], pb[(i + 1) % 2])
        pre_fwd()
    torch.cuda.synchronize()
    with clocked("prefill_stack18_m968"):
        g = capture(pre_fwd, stream)
        ms = time_graph(g, 10, stream)
        del g
        fl = pre[0].flops()
        out["prefill_stack18_m968"] = {"us_per_stack": round(ms * 1e3, 1), "us_per_layer": round(ms * 1e3 / 18, 2),
                                       "tflops": round(18 * fl / (ms * 1e-3) / 1e12, 1),
                                       "frac_fp4_peak": round(18 * fl / (ms * 1e-3) / 1e12 / fp4_peak, 4),
                                       "graph": "18 distinct layers, one CUDA graph"}
    with clocked("prefill_m968"):
        with torch.cuda.stream(stream):
            outs = [nvfp4.empty_fp4(968, 16384, dev) for _ in range(2)]
            ms_gu = gemm_ring_time(pre[0].a2, [p.gate_up for p in pre], "geglu", outs, wsp, stream, reps=10)
            outs_q = [torch.empty((968, 2560), dtype=torch.bfloat16, device=dev) for _ in range(2)]
            ms_q = gemm_ring_time(pre[0].a1, [p.qkv for p in pre], "none", outs_q, wsp, stream, reps=10)
            # down: 64 tiles of 128 x 256 with K = 16384 split in two through the workspace
            outs_d = [torch.empty((968, 2048), dtype=torch.bfloat16, device=dev) for _ in range(2)]
            ms_dn = gemm_ring_time(pre[0].u, [p.down for p in pre], "residual", outs_d, wsp, stream, reps=10,
                                   res=xp)
        tf_gu = 2.0 * 968 * 32768 * 2048 / (ms_gu * 1e-3) / 1e12
        out["prefill_m968"] = {"us_per_layer": out["prefill_stack18_m968"]["us_per_layer"],
                               "tflops": out["prefill_stack18_m968"]["tflops"],
                               "gate_up_us": round(ms_gu * 1e3, 2), "gate_up_tflops": round(tf_gu, 1),
                               "qkv_us": round(ms_q * 1e3, 2),
                               "qkv_tflops": round(2.0 * 968 * 2560 * 2048 / (ms_q * 1e-3) / 1e12, 1),
                               "down_us": round(ms_dn * 1e3, 2),
                               "down_tflops": round(2.0 * 968 * 2048 * 16384 / (ms_dn * 1e-3) / 1e12, 1)}
    # the gate/up GEMM runs as 18 back-to-back launches after a soak, i.e. inside a long step:
    # the sustained peak is the denominator; the burst one is shown beside it
    fp4_sus = pk["bf16_tflops_sustained"] * FP4_OVER_BF16
    out["roofline_m968"] = {"bound": "tensor", "achieved": round(tf_gu, 1), "peak": round(fp4_sus, 1),
                            "unit": "TFLOP/s", "frac": round(tf_gu / fp4_sus, 4),
                            "traffic": traffic("prefill_gate_up"),
                            "algorithmic_bytes_per_launch": gemm_bytes(968, 32768, 2048, "geglu"),
                            "kernel": "gemm_persistent_kernel gate_up 968x32768x2048 GeGLU->FP4",
                            "peak_kind": f"{pk_kind} bf16 sustained x {FP4_OVER_BF16} (nominal fp4/bf16 dense "
                                         "ratio); timed as 18 launches back to back after a soak",
                            "peak_burst": round(fp4_peak, 1), "frac_burst": round(tf_gu / fp4_peak, 4),
                            "clocks": out["prefill_m968"]["clocks"]}
    del pre, xp, pb, outs, outs_q, outs_d
    # ---- M sweep on the 1536 -> 6144 GEMM (bias, bf16 out), 48 distinct weights ----
    with torch.cuda.stream(stream):
        lins = [layers.Linear(synth.bf16_normal_torch(synth.seed_of(5, 1000 + i), (6144, 1536), 0, 0.02,
                                                      device=dev),
                              synth.bf16_normal_torch(synth.seed_of(5, 2000 + i), (6144,), 0, 0.01, device=dev))
                for i in range(48)]
    sweep = []
    with clocked("m_sweep_1536x6144"):
        for Ms in (1, 16, 41, 128, 512, 968):
            with torch.cuda.stream(stream):
                xs = synth.bf16_normal_torch(synth.seed_of(5, Ms), (Ms, 1536), device=dev)
                A = nvfp4.quantize_norm(xs, "none")
                outs = [torch.empty((Ms, 6144), dtype=torch.bfloat16, device=dev) for _ in range(2)]
                ms = gemm_ring_time(A, lins, "bias", outs, wsp, stream, reps=10)
            b = gemm_bytes(Ms, 6144, 1536, "bias")
            gbs = b / (ms * 1e-3) / 1e9
            tf = 2.0 * Ms * 6144 * 1536 / (ms * 1e-3) / 1e12
            # the bound by arithmetic intensity against the ridge of the two measured peaks
            hbm_bound = (2.0 * Ms * 6144 * 1536 / b) < fp4_peak * 1e12 / (pk["hbm_gbs"] * 1e9)
            sweep.append({"M": Ms, "us": round(ms * 1e3, 3), "gbs": round(gbs, 1), "tflops": round(tf, 2),
                          "bound": "hbm" if hbm_bound else "tensor",
                          "frac": round(gbs / pk["hbm_gbs"] if hbm_bound else tf / fp4_peak, 4)})
        out["m_sweep_1536x6144"] = {"points": sweep}
    # ---- norm -> NVFP4 alone at the configs' shapes, over 48 distinct inputs per replay ----
    norm_res = {}
    out["norm_quant"] = norm_res
    with clocked("norm_quant"):
        for label, Mn, Kn, kind in [("adaln_41x1536", 41, 1536, "adaln"),
                                    ("layernorm_41x1536", 41, 1536, "layernorm"),
                                    ("adarms_50x1024", 50, 1024, "adarms"), ("rmsnorm_968x2048", 968, 2048, "rmsnorm")]:
            with torch.cuda.stream(stream):
                xs = [synth.bf16_normal_torch(synth.seed_of(8, 500 + i), (Mn, Kn), device=dev) for i in range(48)]
                gam = synth.bf16_normal_torch(synth.seed_of(8, synth.GAMMA), (Kn,), 1.0, 0.1, device=dev)
                bet = synth.bf16_normal_torch(synth.seed_of(8, synth.BETA), (Kn,), 0.0, 0.1, device=dev)
                sc = synth.bf16_normal_torch(synth.seed_of(8, synth.MOD_SCALE), (Kn,), 0.0, 0.1, device=dev)
                sh = synth.bf16_normal_torch(synth.seed_of(8, synth.MOD_SHIFT), (Kn,), 0.0, 0.1, device=dev)
                prm = {"layernorm": dict(gamma=gam, beta=bet, eps=1e-5), "rmsnorm": dict(gamma=gam, eps=1e-6),
                       "adaln": dict(scale=sc, shift=sh, eps=1e-6), "adarms": dict(scale=sc, eps=1e-6)}[kind]
                qo = nvfp4.empty_fp4(Mn, Kn, dev)

                def norms(xs=xs, kind=kind, prm=prm, qo=qo):
                    for xi in xs:
                        nvfp4.quantize_norm(xi, kind, out=qo, **prm)
                norms()
            torch.cuda.synchronize()
            g = capture(norms, stream)
            ms_n = time_graph(g, 10, stream) / len(xs)
            del g
            nb = 2 * Mn * Kn + Mn * Kn // 2 + Mn * Kn // 16 + 2 * Kn * (2 if kind in ("layernorm", "adaln") else 1)
            norm_res[label] = {"us": round(ms_n * 1e3, 3), "gbs": round(nb / (ms_n * 1e-3) / 1e9, 1), "bytes": nb,
                               "frac_hbm": round(nb / (ms_n * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
            del xs
    # ---- tiny config: LayerNorm->NVFP4 of 41 x 256, then 41 x 512 x 256 GEMM + bias ----
    with torch.cuda.stream(stream):
        tl = [layers.Linear(synth.bf16_normal_torch(synth.seed_of(1, synth.W0 + 100 * i), (512, 256), 0, 0.02,
                                                    device=dev),
                            synth.bf16_normal_torch(synth.seed_of(1, synth.BIAS0 + 100 * i), (512,), 0, 0.01,
                                                    device=dev)) for i in range(48)]
        xt = synth.bf16_normal_torch(synth.seed_of(1, synth.X), (41, 256), device=dev)
        gt = synth.bf16_normal_torch(synth.seed_of(1, synth.GAMMA), (256,), 1.0, 0.1, device=dev)
        bt = synth.bf16_normal_torch(synth.seed_of(1, synth.BETA), (256,), 0.0, 0.1, device=dev)
        at = nvfp4.empty_fp4(41, 256, dev)
        ot = torch.empty((41, 512), dtype=torch.bfloat16, device=dev)

        def tiny():
            for lin in tl:
                nvfp4.quantize_norm(xt, "layernorm", gamma=gt, beta=bt, eps=1e-5, out=at)
                nvfp4.gemm(at, lin.w, "bias", bias=lin.bias, out=ot, workspace=wsp)
        tiny()
    torch.cuda.synchronize()
    with clocked("tiny_41x256_512"):
        g = capture(tiny, stream)
        ms = time_graph(g, 20, stream) / len(tl)
        del g
        # algorithmic bytes of the pair: the norm's x, gamma, beta and FP4 output + the GEMM's
        tb = (2 * 41 * 256 + 4 * 256 + 41 * 128 + 41 * 16) + gemm_bytes(41, 512, 256, "bias")
        gbs_t = tb / (ms * 1e-3) / 1e9
        out["tiny_41x256_512"] = {"us_per_norm_plus_gemm": round(ms * 1e3, 3),
                                  "gemm_bytes": gemm_bytes(41, 512, 256, "bias"),
                                  "roofline": {"bound": "hbm", "achieved": round(gbs_t, 1), "peak": pk["hbm_gbs"],
                                               "unit": "GB/s", "frac": round(gbs_t / pk["hbm_gbs"], 4),
                                               "bytes": tb, "peak_kind": pk_kind},
                                  "l2": "48 distinct weight copies (L2-warm: 3.6 MB in total)"}
    # ---- the block-scaled MMA's issue rate on one SM (nvfp4_mma_rate): the ceiling of the
    # GEMM kernels' MMA phases; cycles per K step of 256 (4 MMAs of 128 x n x 64), MMAs alone
    # (mode 0) and with the step's scale-atom copies from the same thread (mode 1) ----
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    rate = {}
    out["mma_rate"] = rate
    with clocked("mma_rate"):
        for n in (64, 128, 256):
            _, c0 = nvfp4.mma_rate(n, 0, 256)
            _, c1 = nvfp4.mma_rate(n, 1, 256)
            flop_per_cycle = 4 * 2.0 * 128 * n * 64 / c0
            rate[f"n{n}"] = {"mma_cycles_per_kstep": round(c0, 1), "copies_and_mma_cycles_per_kstep": round(c1, 1),
                             "fp4_flop_per_sm_cycle": round(flop_per_cycle, 1)}
    max_mhz = rate["clocks"].get("sm_max_mhz") or 0.0
    rate["implied_fp4_tflops_at_max_clock"] = round(rate["n256"]["fp4_flop_per_sm_cycle"] * sms * max_mhz * 1e6 / 1e12,
                                                    1)
    rate["note"] = ("one CTA, one issuing thread, operands resident in shared memory; the implied figure is the "
                    "256-wide MMA rate x SMs x the maximum SM clock, context for the FP4 peak, not its denominator")
    torch.cuda.synchronize()
    nvfp4.device_status()
    return out


if __name__ == "__main__":
    sys.exit(main())
