"""Benchmark of the CSA/HCA hot path on B200: decode queries/s and roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c1] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
for a CSA workload csa_compress (the block the step completes) ->
csa_index_topk -> csa_sparse_attn; for an HCA workload hca_compress ->
hca_dense_attn.  The default workload is the V4-Flash-shaped CSA decode
(batch 32, 131072-token context, 32768 entries, top-512, 64 heads).

Timing: W untimed warm-up steps, then exactly K steps between CUDA events on
the launching stream, bracketed by a barrier and torch.cuda.synchronize().
In a CSA step the compressor runs on a forked stream beside the index call
(the two are independent; the attention waits for both).
The timed loop rotates over several device-resident copies of the workload
so that the bytes one cycle touches exceed 3x the L2 size: every step reads
its inputs from HBM, no flush is needed.  Multi-GPU (torchrun): every rank
runs the same per-GPU workload (weak scaling) with no data-path collective;
the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only other program here that
runs the same method) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "CSA/HCA decode queries/s at 128K-1M ctx; % of HBM / tensor-core roofline"
L2_BYTES = 126 * 2 ** 20

CONFIG_NAMES = {
    "c0": "tiny CSA decode fp32 (B=1, L=2048, d=128)",
    "c1": "V4-Flash-shaped CSA decode (B=32, L=131072, N=32768, top-512, n_h=64, d=512 FP8+BF16, MXFP4 indexer 64x128)",
    "c2": "V4-Pro-shaped CSA decode (B=4, L=1048576, N=262144, top-1024, n_h=128, planted cluster)",
    "c3": "HCA decode (B=16, L=1048576, m=128, N=8192, n_h=128, dense)",
    "c4": "CSA chunked prefill (B=2, T=32768, N=8192, top-512, n_h=64)",
}


def algorithmic_bytes(w):
    """Bytes the method must move per step, and those of the dominant call.

    Per query of a CSA decode: every visible index key (c/2 + c/32 bytes),
    the index query + weights, the k selected entries and W window rows
    (d + r + 4 bytes each), the query and the output (n_h*d*2 each), the
    k indices; plus the compressor's 2m stream rows and gates and its
    written entry.  HCA: every visible entry instead of keys/selection.
    Returns (step_bytes, index_call_bytes).
    """
    p = w["params"]
    B, T = p.B, w["T"]
    row = p.d + p.r + 4 if p.kv_fmt == "fp8" else 4 * p.d
    act = 2 if p.act_fmt == "bf16" else 4
    key = p.c_I // 2 + p.c_I // 32 if p.idx_fmt == "mxfp4" else 4 * p.c_I
    step = idx_call = 0
    for b in range(B):
        for tq in range(T):
            t = int(w["q_pos0"][b]) + tq
            n_t = min((t + 1) // p.m, w["Ncap"])
            win = min(p.W, t + 1)
            qo = 2 * p.n_h * p.d * act
            if p.k > 0:
                iq = p.H_I * key + 4 * p.H_I
                ic = n_t * key + iq + 4 * p.k
                idx_call += ic
                step += ic + (min(p.k, n_t) + win) * row + qo + 4 * p.k
            else:
                step += (n_t + win) * row + qo
    if w["S"]:
        ne = int((np.asarray(w["e_end"]) - np.asarray(w["e_begin"])).sum())
        step += ne * (2 * p.m * p.d * act + 2 * p.m * 4 + row + 4)
    return step, idx_call


def algorithmic_flops(w):
    """Tensor work of the attention per step: for every query, head and
    attended row (top-k entries or every visible entry, plus the window),
    q.v (2d flops) and p*v (2d flops)."""
    p = w["params"]
    B, T = p.B, w["T"]
    total = 0
    for b in range(B):
        for tq in range(T):
            t = int(w["q_pos0"][b]) + tq
            n_t = min((t + 1) // p.m, w["Ncap"])
            rows = (min(p.k, n_t) if p.k > 0 else n_t) + min(p.W, t + 1)
            total += p.n_h * rows * 4 * p.d
    return total


def index_flops(w):
    """Lightning Indexer multiply-adds per step (MXFP4 contraction): 2 H_I c_I
    flops per (query, visible entry)."""
    p = w["params"]
    total = 0
    if p.k <= 0:
        return 0
    for b in range(p.B):
        for tq in range(w["T"]):
            t = int(w["q_pos0"][b]) + tq
            total += 2 * p.H_I * p.c_I * min((t + 1) // p.m, w["Ncap"])
    return total


FP4_OVER_BF16 = 4.0  # nominal dense ratio of B200's FP4 and BF16 tensor rates (9 / 2.25 PFLOP/s)

_PEAK_CACHE = {}


def probe_tensor_peak(kind):
    """Dense tcgen05.mma throughput measured live on this GPU by the probe
    library (every SM issuing back-to-back M=128, N=256 MMAs; best of 5
    launches): kind "mxf4" (E2M1, block-scaled) or "bf16".  TFLOP/s, or None
    if the probe fails."""
    if kind in _PEAK_CACHE:
        return _PEAK_CACHE[kind]
    val = None
    try:
        import ctypes
        from long_context_sparse_gated_b200 import build
        L = ctypes.CDLL(build.build_peak())
        L.csa_peak_mma_tflops.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.csa_peak_mma_tflops.restype = ctypes.c_double
        v = L.csa_peak_mma_tflops(0 if kind == "mxf4" else 1, 20000, 5)
        val = v if v > 0 else None
    except Exception:
        val = None
    _PEAK_CACHE[kind] = val
    return val


def fp4_peak(bf16_peak, bf16_src):
    """The MXFP4 dense peak: measured by the probe, else the BF16 peak times
    the nominal ratio (said so in the source string)."""
    v = probe_tensor_peak("mxf4")
    if v is not None:
        return v, "measured live: tcgen05.mma kind::mxf4 M=128 N=256 K=64, all SMs, best of 5 (bench.py probe)"
    return bf16_peak * FP4_OVER_BF16, f"{bf16_src} bf16 x {FP4_OVER_BF16:g} (nominal fp4:bf16)"


def dominant_roofline(w, kmean_ms, amean_ms, idx_bytes, step_bytes, hbm, bf16, traffic):
    """Roofline entry of the step's dominant call.  hbm = (GB/s, source) and
    bf16 = (TFLOP/s, source) are the measured peaks.

    The dominant call is the one that takes longer of the index call
    (kmean_ms) and the attention (amean_ms; for HCA the dense attention is
    the only timed call).  CSA decode: the index call streams every visible
    key once, HBM-bound.  CSA prefill: the index call's MXFP4 contraction is
    tensor-bound (peak: the FP4 peak measured live); the sparse attention,
    4d flops per (head, attended row), is tensor-bound (BF16 peak; FP16
    operands run at the BF16 rate).  HCA: the dense attention, likewise."""
    p = w["params"]
    sec = kmean_ms * 1e-3
    hbm_peak, hbm_src = hbm
    bf16_peak, bf16_src = bf16
    dom_bytes = idx_bytes if p.k > 0 else step_bytes
    hbm_ach = dom_bytes / sec / 1e9
    if p.k > 0:
        fl = index_flops(w)
        fp4_pk, fp4_src = fp4_peak(bf16_peak, bf16_src)
        fp4_ach = fl / sec / 1e12
        if w["T"] <= 4:
            return {"bound": "hbm", "kernel": "csa_index_topk", "achieved": hbm_ach, "peak": hbm_peak,
                    "unit": "GB/s", "frac": hbm_ach / hbm_peak, "peak_source": hbm_src, "traffic": traffic,
                    "frac_vs_8tbs_datasheet": hbm_ach / 8000.0,
                    "algorithmic_bytes_per_launch": dom_bytes, "launch_ms": kmean_ms,
                    "fp4_tflops": fp4_ach, "fp4_peak": fp4_pk, "fp4_frac": fp4_ach / fp4_pk,
                    "fp4_peak_source": fp4_src}
        idx = {"bound": "tensor", "kernel": "csa_index_topk", "achieved": fp4_ach, "peak": fp4_pk,
               "unit": "TFLOP/s", "frac": fp4_ach / fp4_pk,
               "peak_source": fp4_src, "traffic": traffic,
               "algorithmic_flops_per_launch": fl, "launch_ms": kmean_ms,
               "hbm_achieved_gbs": hbm_ach, "hbm_frac": hbm_ach / hbm_peak}
        if amean_ms <= kmean_ms:
            return idx
        fa = algorithmic_flops(w)
        a_ach = fa / (amean_ms * 1e-3) / 1e12
        return {"bound": "tensor", "kernel": "csa_sparse_attn", "achieved": a_ach, "peak": bf16_peak,
                "unit": "TFLOP/s", "frac": a_ach / bf16_peak, "peak_source": bf16_src, "traffic": None,
                "algorithmic_flops_per_launch": fa, "launch_ms": amean_ms, "index_call": idx}
    fl = algorithmic_flops(w)
    ach = fl / sec / 1e12
    return {"bound": "tensor", "kernel": "hca_dense_attn", "achieved": ach, "peak": bf16_peak,
            "unit": "TFLOP/s", "frac": ach / bf16_peak, "peak_source": bf16_src, "traffic": None,
            "algorithmic_flops_per_launch": fl, "launch_ms": kmean_ms,
            "hbm_achieved_gbs": hbm_ach, "hbm_frac": hbm_ach / hbm_peak}


def step_roofline_entry(w, ms_per_step, step_bytes, hbm_peak, bf16_peak):
    """The whole step against both roofs: its algorithmic bytes over the HBM
    peak, and its two contractions (the indexer's MXFP4 flops, the
    attention's BF16/FP16 flops) over their tensor peaks, all over the step
    time."""
    sec = ms_per_step * 1e-3
    gbs = step_bytes / sec / 1e9
    fl_i, fl_a = index_flops(w), algorithmic_flops(w)
    fp4_pk = fp4_peak(bf16_peak, "")[0]
    return {"algorithmic_bytes": step_bytes, "achieved_gbs": gbs, "frac": gbs / hbm_peak,
            "index_fp4_tflops": fl_i / sec / 1e12, "index_fp4_frac": fl_i / sec / 1e12 / fp4_pk,
            "attn_tflops": fl_a / sec / 1e12, "attn_bf16_frac": fl_a / sec / 1e12 / bf16_peak}


def launches_per_step(w):
    """Kernels one step enqueues (the fallback when the captured graphs'
    kernel nodes cannot be counted): compress, scorer, selector (plus the
    chunked candidate pass for rows over 32768 entries), attention (plus the
    split merge in decode)."""
    p = w["params"]
    n = 1 if w["S"] else 0
    if p.k > 0:
        hist = w["T"] * p.B <= 4096
        n_max = int(min(w["Ncap"], ((np.asarray(w["q_pos0"]) + w["T"]) // p.m).max()))
        n += 2 + (1 if hist and n_max > 32768 else 0)
        n += 2 if w["T"] <= 4 else 1
    else:
        n += 2 if w["T"] <= 4 else 1
    return n


def graph_kernel_nodes(graph):
    """Kernel nodes of a captured CUDA graph (driver API on the raw handle);
    None when the handle or the driver call is not available."""
    try:
        import ctypes
        drv = ctypes.CDLL("libcuda.so.1")
        h = ctypes.c_void_p(graph.raw_cuda_graph())
        n = ctypes.c_size_t(0)
        if drv.cuGraphGetNodes(h, None, ctypes.byref(n)) != 0:
            return None
        nodes = (ctypes.c_void_p * n.value)()
        if drv.cuGraphGetNodes(h, nodes, ctypes.byref(n)) != 0:
            return None
        kernels = 0
        for i in range(n.value):
            t = ctypes.c_int(-1)
            if drv.cuGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(t)) != 0:
                return None
            kernels += t.value == 0  # CU_GRAPH_NODE_TYPE_KERNEL
        return kernels
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out = self.proc.communicate(timeout=10)[0]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def recorded_traffic(key):
    """DRAM bytes per launch of the dominant call from the committed ncu
    capture (profiles/dram_traffic.json), or None when the kernels' sources
    changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            e = json.load(f)[key]
        h = hashlib.sha1()
        for src in e["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        return int(e["bytes_per_launch"]) if h.hexdigest() == e["sources_sha1"] else None
    except (OSError, KeyError, ValueError):
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense BF16 tensor peak (burst: the kernel is timed by events around
    one call, not over seconds); FP16 operands run at the same rate."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def sample_queries(w, config):
    """The bounded sample of queries the oracle is timed on, and its
    description.  Decode: the first few queries.  Prefill: a stratified
    sample of sequence 0's positions (the oracle's cost grows with the
    position): the first 16, 16 around t = 2047, the last 16 and 16 seeded
    uniform others."""
    p = w["params"]
    T = w["T"]
    if T <= 4:
        n = CPU_SAMPLE[config]
        return [(b, tq) for b in range(p.B) for tq in range(T)][:n], f"first {n} queries of the workload"
    pos = set(range(16)) | set(range(max(0, 2040), min(T, 2056))) | set(range(T - 16, T))
    rest = np.setdiff1d(np.arange(T), np.fromiter(pos, dtype=np.int64))
    pos |= set(int(x) for x in np.random.default_rng(12345).choice(rest, size=min(16, len(rest)), replace=False))
    qs = [(0, int(tq)) for tq in sorted(pos)]
    return qs, (f"{len(qs)} positions of sequence 0: first 16, 16 around t=2047, last 16, 16 seeded uniform")


def oracle_sample(w, queries):
    """Time the oracle on the given queries of the workload."""
    from oracle import pipeline
    p = w["params"]
    qs = list(queries)
    seqs = sorted(set(b for b, _ in qs))
    t0 = time.perf_counter()
    comp = pipeline.compress(w, seqs=seqs) if w["S"] else None
    if p.k > 0:
        idx = pipeline.index_topk(w, qs)
        pipeline.sparse_attn(w, idx, comp, qs)
    else:
        pipeline.dense_attn(w, comp, qs)
    return time.perf_counter() - t0, len(qs)


CPU_SAMPLE = {"c0": 1, "c1": 4, "c2": 1, "c3": 4, "c4": 16}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline_entry(w, config):
    """The oracle on a bounded sample of the workload (its first queries),
    with the host threads its numpy/BLAS pool uses, then with one thread."""
    qs, what = sample_queries(w, config)
    dt, nq = oracle_sample(w, qs)
    entry = {"value": nq / dt, "unit": "queries/s", "cores": cpu_cores(), "kind": "oracle",
             "sample": f"{what} (numpy fp64 oracle, {dt:.1f} s)",
             "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            dt1, nq1 = oracle_sample(w, qs)
        entry["value_1_thread"] = nq1 / dt1
    except Exception:
        pass
    return entry


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


CONFIG_SEEDS = {"c0": 0, "c1": 1, "c2": 2, "c3": 3, "c4": 4}


def rank_seed(config, rank):
    """Weak scaling: every rank runs the same per-GPU workload shape, drawn
    from its own seed (no data-path exchange between ranks)."""
    return CONFIG_SEEDS[config] + 1000 * rank


def max_over_ranks(values, device):
    """Element-wise max of each rank's timings over all ranks of the default
    process group (every rank must call it, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_value(world, queries_per_rank, ms_per_step):
    """Whole-job throughput: the queries all ranks processed per second of
    the slowest rank's step time."""
    return world * queries_per_rank / (ms_per_step * 1e-3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.config(args.config)
    qs, what = sample_queries(w, args.config)
    n = len(qs)
    for _ in range(args.warmup and 1):
        oracle_sample(w, qs[:1])
    times = []
    for _ in range(args.steps):
        dt, nq = oracle_sample(w, qs)
        times.append(dt)
    total = sum(times)
    qps = args.steps * n / total
    line = {"impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": CONFIG_NAMES[args.config], "name": args.config,
                                            "sample_queries_per_step": n},
            "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": f"{what} per step (oracle: numpy fp64)", "cpu_model": cpu_model(),
                             "nproc": os.cpu_count()},
            "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="c1", choices=sorted(CONFIG_NAMES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every call from the host (no CUDA graphs)")
    ap.add_argument("--copies", type=int, default=0,
                    help="device copies rotated in the timed loop (0: enough to exceed 3x L2)")
    ap.add_argument("--score-fmt", default="f32", choices=["f32", "bf16"],
                    help="index-score precision the selector ranks (bf16: the BF16-score variant)")
    ap.add_argument("--prefill-len", type=int, default=0,
                    help="c4 only: a shorter prefill (L = T = this many tokens per sequence) for profiling "
                         "small cases; 0 keeps the workload's 32768")
    ap.add_argument("--extra-configs", default="c2,c3,c4",
                    help="with --config c1 on one GPU: the other workloads measured into the same line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from long_context_sparse_gated_b200 import build, lib
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        dist.barrier()
    lib()

    names = [args.config]
    if world == 1 and args.config == "c1":
        names += [c for c in args.extra_configs.split(",") if c and c != args.config]
    lines = {}
    for name in names:
        lines[name] = run_config(name, args, world, rank, local)
        torch.cuda.empty_cache()
    if rank == 0:
        line = lines[names[0]]
        if len(names) > 1:
            # the other workloads of the same metric, each measured the same
            # way (its own roofline, clocks, end-to-end and CPU baseline)
            line["configs"] = {n: lines[n] for n in names[1:]}
        line["tensor_peaks_measured"] = {"mxf4_tflops": probe_tensor_peak("mxf4"),
                                         "bf16_tflops": probe_tensor_peak("bf16"),
                                         "how": "tcgen05.mma M=128 N=256 back to back from one thread per SM, all SMs, "
                                                "best of 5 launches of 20000 MMAs (burst)"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def bf16_score_entry(w, dw32, stream, reps=20):
    """The BF16-score variant of the index call on the same inputs (kwkr.cn
    notes 4.4: index scores quantised from FP32 to BF16 before the top-k
    selector): its mean event time beside the fp32 call's, and how much of
    the fp32-score top-k set the BF16-score selection keeps (mean over the
    batch's queries).  Both sets are exact (tests compare each with the
    oracle's selection), so this is the recall of the method, not of the
    kernels."""
    import torch
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw16 = DeviceWorkload(synth.with_score_fmt(w, "bf16"))

    def timed(dw):
        for _ in range(3):
            dw.index_topk()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dw.index_topk()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return float(np.median(ts)) * 1e3

    us32, us16 = timed(dw32), timed(dw16)
    i32 = dw32.idx.cpu().numpy().reshape(-1, dw32.idx.shape[-1])
    i16 = dw16.idx.cpu().numpy().reshape(-1, dw16.idx.shape[-1])
    rec = []
    for a, b in zip(i32, i16):
        sa = set(a[a >= 0].tolist())
        rec.append(len(sa & set(b[b >= 0].tolist())) / max(len(sa), 1))
    del dw16
    return {"index_call_us_fp32": us32, "index_call_us_bf16": us16,
            "recall_of_fp32_topk": float(np.mean(rec)), "recall_min": float(np.min(rec)),
            "how": "host-launched index calls on one device copy, median of 20 event-timed calls each; "
                   "recall = |BF16-score top-k & fp32-score top-k| / min(k, n_t), mean over the queries"}


def host_call_us(dw, reps=100):
    """Host time per public call through the Python binding: the mean wall
    time of `reps` back-to-back calls, with the device work queued behind
    and not waited for (argument checks, cached driver work, launches)."""
    import torch
    calls = {"csa_compress" if dw.p.m < 64 else "hca_compress": dw.compress}
    if dw.p.k > 0:
        calls.update({"csa_index_topk": dw.index_topk, "csa_sparse_attn": dw.sparse_attn})
    else:
        calls["hca_dense_attn"] = dw.dense_attn
    out = {}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        t = time.perf_counter()
        for _ in range(reps):
            fn()
        out[name] = (time.perf_counter() - t) / reps * 1e6
        torch.cuda.synchronize()
    out["how"] = f"mean wall time of {reps} back-to-back host calls, device work not awaited"
    return out


def run_config(config, args, world, rank, local):
    """Measure one workload; rank 0 returns its JSON entry, others None."""
    import torch
    import torch.distributed as dist
    from long_context_sparse_gated_b200.runner import STEP_INPUTS, DeviceWorkload

    over = {"L": args.prefill_len} if config == "c4" and args.prefill_len > 0 else {}
    w = synth.with_score_fmt(synth.config(config, seed=rank_seed(config, rank), **over), args.score_fmt)
    step_bytes, idx_bytes = algorithmic_bytes(w)
    n_copies = max(1, int(np.ceil(3 * L2_BYTES / step_bytes)))
    if config == "c4":
        n_copies = 1  # prefill touches far more than L2 per step
    if args.copies > 0:
        n_copies = args.copies
    dws = [DeviceWorkload(w) for _ in range(n_copies)]
    p = w["params"]
    queries = p.B * w["T"]
    stream = torch.cuda.current_stream()

    side0 = torch.cuda.Stream()

    def step(dw, ev=None):
        if p.k > 0:
            # the compressor runs beside the index call (independent)
            side0.wait_stream(stream)
            with torch.cuda.stream(side0):
                dw.compress(side0)
            if ev is not None:
                ev[0].record(stream)
            dw.index_topk()
            if ev is not None:
                ev[1].record(stream)
            stream.wait_stream(side0)
            dw.sparse_attn()
            if ev is not None:
                ev[2].record(stream)
        else:
            dw.compress()
            if ev is not None:
                ev[0].record(stream)
            dw.dense_attn()
            if ev is not None:
                ev[1].record(stream)

    for i in range(args.warmup):
        step(dws[i % n_copies])
    torch.cuda.synchronize()

    # Each copy's step is captured as CUDA graphs so that host launch cost
    # does not starve the device; events between the replays time the
    # dominant call.  CSA: the compressor and the index call are independent
    # (only the attention reads the new entry), so one graph runs the
    # compressor on a forked branch concurrently with the index call (the
    # events around it then time the index call with the compressor
    # running beside it), a second graph the attention.  HCA: compress, then
    # the dense attention (dependent).
    graphs = []
    kernels_per_step = None  # counted from the captured graphs when possible
    if not args.no_graph:
        cap = torch.cuda.Stream()
        side = torch.cuda.Stream()
        cap.wait_stream(stream)

        def fork_compress_index(dw):
            def run(st):
                side.wait_stream(st)
                with torch.cuda.stream(side):
                    dw.compress(side)
                dw.index_topk(st)
                st.wait_stream(side)
            return run

        for dw in dws:
            phases = [None, fork_compress_index(dw), dw.sparse_attn] if p.k > 0 else [dw.compress, dw.dense_attn, None]
            parts = []
            with torch.cuda.stream(cap):
                for fn in phases:
                    g = None
                    if fn is not None:
                        try:
                            g = torch.cuda.CUDAGraph(keep_graph=True)
                        except TypeError:
                            g = torch.cuda.CUDAGraph()
                        with torch.cuda.graph(g, stream=cap):
                            fn(cap)
                    parts.append(g)
            graphs.append(parts)
        stream.wait_stream(cap)
        torch.cuda.synchronize()
        counts = [graph_kernel_nodes(g) for g in graphs[0] if g is not None]
        if counts and all(c is not None for c in counts):
            kernels_per_step = sum(counts)

    def timed_step(i, ev=None):
        if not graphs:
            return step(dws[i % n_copies], ev)
        g0, g1, g2 = graphs[i % n_copies]
        if g0 is not None:
            g0.replay()
        if ev is not None:
            ev[0].record(stream)
        g1.replay()
        if ev is not None:
            ev[1].record(stream)
        if g2 is not None:
            g2.replay()
            if ev is not None:
                ev[2].record(stream)

    for i in range(3):
        timed_step(i)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    # keep the GPU busy while the sampler starts (untimed)
    t_end = time.perf_counter() + 0.5
    i = 0
    while time.perf_counter() < t_end:
        timed_step(i)
        i += 1
    torch.cuda.synchronize()

    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        timed_step(i, evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    kern_ms = [e[0].elapsed_time(e[1]) for e in evs]
    # CSA: the sparse attention (its graph replays right after the index call's)
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs] if p.k > 0 else kern_ms
    # a little more load for the clock sampler, then stop it (untimed)
    t_end = time.perf_counter() + 0.3
    while time.perf_counter() < t_end:
        timed_step(i)
        i += 1
    torch.cuda.synchronize()
    clocks = sampler.stop()
    del graphs

    # ---- end to end: per-step inputs from pinned host memory, results back --
    # A serving pipeline over two buffer sets: step i's inputs are copied in
    # on a copy stream while step i-1 computes, and step i's output and
    # indices are read back on another copy stream while step i+1 computes.
    # Every step still copies all of its inputs in and its results out inside
    # the timed region; only the overlap across steps is new.
    nb = 2 if n_copies >= 2 else 1
    bufs = dws[:nb]
    host_in = [{k: getattr(d, k).cpu().pin_memory() for k in STEP_INPUTS if getattr(d, k, None) is not None}
               for d in bufs]
    host_out = [d.out.cpu().pin_memory() for d in bufs]
    host_idx = [d.idx.cpu().pin_memory() for d in bufs]
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = host_out[0].numel() * host_out[0].element_size() + (host_idx[0].numel() * 4 if p.k > 0 else 0)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in bufs]
    ev_done = [torch.cuda.Event() for _ in bufs]
    ev_out = [torch.cuda.Event() for _ in bufs]

    def e2e_step(i):
        j = i % nb
        d = bufs[j]
        if i >= nb:
            s_in.wait_event(ev_done[j])  # step i-nb has consumed buffer j's inputs
        with torch.cuda.stream(s_in):
            for k, t in host_in[j].items():
                getattr(d, k).copy_(t, non_blocking=True)
        ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= nb:
            stream.wait_event(ev_out[j])  # step i-nb's results have been read back
        step(d)
        ev_done[j].record(stream)
        s_out.wait_event(ev_done[j])
        with torch.cuda.stream(s_out):
            host_out[j].copy_(d.out, non_blocking=True)
            if p.k > 0:
                host_idx[j].copy_(d.idx, non_blocking=True)
        ev_out[j].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(10, min(args.steps, 200))
    e0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e

    kmean = float(np.mean(kern_ms))
    amean = float(np.mean(attn_ms))
    if world > 1:
        ms, e2e_ms, kmean, amean = max_over_ranks([ms, e2e_ms, kmean, amean], "cuda")
    err = int(sum(d.err_bits() for d in dws))

    if rank != 0:
        del dws
        return None
    ms_per_step = ms / args.steps
    value = job_value(world, queries, ms_per_step)
    peak, peak_kind = measured_peaks()
    roofline = dominant_roofline(w, kmean, amean, idx_bytes, step_bytes, (peak, peak_kind), measured_tensor_peak(),
                                 recorded_traffic(f"csa_index_topk@{config}") if p.k > 0 else None)
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8/bf16 storage, mxfp4 indexer, fp32 accumulate" if p.kv_fmt == "fp8" else "f32",
        "data": "synthetic",
        "config": {"workload": CONFIG_NAMES[config] + (f", reduced to L = T = {args.prefill_len}" if over else ""),
                   "name": config, "batch": p.B, "index_scores": args.score_fmt,
                   "context": int(w["L"].max()), "queries_per_step": queries,
                   "l2": f"inputs larger than L2: {n_copies} device copies rotated, {n_copies * step_bytes / 2**20:.0f} MiB per cycle"},
        "gpu_launches": args.steps * (kernels_per_step if kernels_per_step is not None else launches_per_step(w)),
        "gpu_launches_source": "graph kernel nodes" if kernels_per_step is not None else "static count",
        "graphs": not args.no_graph,
        "roofline": roofline,
        "calls_ms": ({"index_call_with_compress_beside": kmean, "attention": amean} if p.k > 0
                     else {"dense_attention": kmean}),
        "step_roofline": step_roofline_entry(w, ms_per_step, step_bytes, peak, measured_tensor_peak()[0]),
        "e2e": {"value": job_value(world, queries, e2e_ms), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clocks,
        "device_err_bits": err,
    }
    if world == 1:
        line["host_us_per_call"] = host_call_us(dws[0], reps=100 if queries <= 4096 else 10)
    if p.k > 0 and w["T"] <= 4 and args.score_fmt == "f32" and world == 1:
        line["bf16_scores"] = bf16_score_entry(w, dws[0], stream)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline_entry(w, config)
    del dws
    return line


if __name__ == "__main__":
    main()
