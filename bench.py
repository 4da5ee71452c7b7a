"""Benchmark of the W4A8 linear layer on B200: TOPS and % of roofline vs M.

One step = one pass of the whole hot path -- per-token activation
quantization, then the W4A8 GEMM with its epilogue -- over every shape of the
workload, with weights packed offline (untimed) and resident in HBM.

The default workload is the Llama-3-8B MLP up-projection at decode batch
sizes: M in {1, 8, 32, 64}, K = 4096, N = 14336, per-channel and g128
weights (8 GEMMs per step).  `--workload sweep|large_batch|qwen|tiny` selects
the other workloads for ad-hoc measurement.

Timing: when the distinct packed weights of a step exceed 1.5x L2
(126 MB; the decode workload holds 224 MB), the shapes run back to back and
the step is bracketed by CUDA events on the launching stream: every weight
byte comes from HBM, because the step has cycled more than L2 since it last
read the same weights.  Smaller workloads flush L2 (a 256 MB write) before
every shape instead, bracket each shape with events (flush excluded) and sum.
K timed steps follow W untimed ones, bracketed by a barrier and a device
synchronize; with N > 1 every rank runs the same workload (replicas, weak
scaling) and the time is the max over ranks.  Per shape, an isolated run
(L2 flushed, the kernels alone) gives the per-point breakdown.

--impl reference times the CPU oracle (plain C, OpenMP) on a bounded sample
of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from w4a8_integer_gemm_b200 import roofline, workloads as wl  # noqa: E402

FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20
GEMM_SOURCES = ("qoq_gemm.cu", "qoq_layout.cuh", "qoq_ptx.cuh", "qoq_internal.h", "qoq_quant.cuh")


def code_only(text: str) -> str:
    """C/C++ source as the library build compiles it, for hashing: without
    comments, without the trace build's `#ifdef QOQ_TRACE` branches (their
    `#else` branches stay), and with whitespace collapsed.  A change of
    wording or of trace-only code leaves the hash as it was."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    kept, stack = [], []  # stack: per open #if, whether we are in its trace-only branch
    for line in text.splitlines():
        d = line.strip()
        if d.startswith("#if"):
            stack.append(d.split()[:2] == ["#ifdef", "QOQ_TRACE"])
        elif d.startswith("#else") or d.startswith("#elif"):
            if stack:
                stack[-1] = False
        elif d.startswith("#endif"):
            if stack:
                stack.pop()
        elif not any(stack):
            kept.append(line)  # conditional directives themselves are not kept
    return " ".join(" ".join(kept).split())


def gemm_source_hash(read=None) -> str:
    """Short hash of the GEMM kernel's code (comments excluded): DRAM traffic
    recorded under profiles/ is reported only while it matches, since the
    counters describe that kernel and no later one.  `read(name)` returns a
    source file's text (default: the working tree)."""
    import hashlib
    if read is None:
        def read(f):
            with open(os.path.join(ROOT, "w4a8_integer_gemm_b200", "csrc", f)) as fh:
                return fh.read()
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(code_only(read(f)).encode())
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--only", default=None,
                    help="restrict the workload to one shape name (for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every kernel from Python in the timed steps instead of replaying a CUDA graph")
    ap.add_argument("--a-smem", action="store_true",
                    help="keep the GEMM's dequantized tile in shared memory instead of TMEM")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample (cpu_baseline / reference arm)")
    return ap.parse_args()


def select(args) -> wl.Workload:
    work = wl.WORKLOADS[args.workload]
    if args.only:
        keep = [s for s in work.shapes if s.name == args.only]
        if not keep:
            raise SystemExit(f"no shape {args.only!r} in {work.name}")
        idx = work.shapes.index(keep[0])
        # keep the shape's own seeds: a one-shape workload with the same number
        sub = wl.Workload(work.number, work.name, work.dist, list(work.shapes))
        sub.shapes = [work.shapes[idx]]
        sub.seeds = lambda i, _w=work, _k=idx: _w.seeds(_k)
        return sub
    return work


# ----------------------------------------------------------- distributed --
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return rank, world, local, dist
    return rank, world, local, None


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(x: float, dist) -> float:
    if dist is None:
        return x
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(ops_per_rank: float, ms_this_rank: float, world: int, dist):
    """Whole-job throughput of `world` replicas that each did ops_per_rank
    operations: the step time is the slowest rank's (max over ranks), the
    value is all ranks' operations over that time, in TOPS."""
    ms = max_over_ranks(ms_this_rank, dist)
    return ms, world * ops_per_rank / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9 and p[1].isdigit():
                    rows.append(p)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3] != "[N/A]")}


# --------------------------------------------------------------- our arm --
def run_ours(args, rank, world, local, dist):
    import w4a8_integer_gemm_b200 as q

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q.lib()
    q.qoq_set_gemm_a_in_tmem(not args.a_smem)
    peaks = roofline.load_peaks()
    work = select(args)
    stream = torch.cuda.current_stream()

    # inputs: seeded synthetic draws, packed offline, resident in HBM
    cases = []
    for i, s in enumerate(work.shapes):
        X, W = wl.make_case(work, i)
        packed = q.qoq_pack_weights(W.to(dev), s.G)
        Xd = X.to(dev)
        X8 = torch.empty(s.M, s.K, dtype=torch.int8, device=dev)
        s_x = torch.empty(max(s.M, 8), dtype=torch.int16, device=dev)
        Y = torch.empty(s.M, s.N, dtype=torch.float16, device=dev)
        ws = torch.zeros(q.qoq_gemm_workspace_bytes(s.M, s.N, s.K, s.G), dtype=torch.uint8, device=dev)
        Xh = X.pin_memory()
        Yh = torch.empty(s.M, s.N, dtype=torch.float16, pin_memory=True)
        cases.append(dict(s=s, packed=packed, X=Xd, X8=X8, s_x=s_x, Y=Y, ws=ws, Xh=Xh, Yh=Yh))
        del W
    torch.cuda.synchronize()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n_sh = len(cases)
    wbytes = sum(c["packed"].Wp.numel() for c in cases)
    # Each step touches every shape's own packed weights once.  When they
    # add up to more than 1.5x the L2 (126 MB) the step runs back to back,
    # as a serving stack would run consecutive layers, and the weights of a
    # shape are long evicted before the next step comes back to them.
    # Otherwise L2 is flushed before every shape and each shape is timed
    # on its own (flush excluded).
    chained = wbytes > 3 * L2_BYTES // 2
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [[E() for _ in range(4)] for _ in range(n_sh)]
    es = [E(), E(), E(), E()]

    def enqueue_step(st, gemm=True, quant=True, fused=True):
        """Launch the step's kernels on stream st: per shape the layer call
        (qoq_w4a8_linear), or the quantizer and the GEMM as separate calls."""
        for c in cases:
            if quant and gemm and fused:
                q.qoq_w4a8_linear(c["X"], c["packed"], X8=c["X8"], s_x=c["s_x"], Y=c["Y"], workspace=c["ws"],
                                  stream=st)
                continue
            if quant:
                q.qoq_quant_act_per_token(c["X"], c["X8"], c["s_x"], stream=st)
            if gemm:
                q.qoq_w4a8_gemm(c["X8"], c["s_x"], c["packed"], Y=c["Y"], workspace=c["ws"], stream=st)

    graphs = {}

    def one_step(eager=False):
        """The hot path of every shape: activation quant, then the GEMM.
        Returns the step's device time in ms."""
        if chained:
            es[0].record(stream)
            if "step" in graphs and not eager:
                graphs["step"].replay()
            else:
                enqueue_step(stream)
            es[1].record(stream)
            torch.cuda.synchronize()
            return es[0].elapsed_time(es[1])
        for j, c in enumerate(cases):
            flush.zero_()
            ev[j][0].record(stream)
            q.qoq_w4a8_linear(c["X"], c["packed"], X8=c["X8"], s_x=c["s_x"], Y=c["Y"], workspace=c["ws"],
                              stream=stream)
            ev[j][1].record(stream)
        torch.cuda.synchronize()
        return sum(ev[j][0].elapsed_time(ev[j][1]) for j in range(n_sh))

    def one_launch_step():
        """The same step with the layer call as one GEMM launch that
        quantizes its own rows (replayed from a graph when chained), for
        comparison."""
        if chained:
            es[0].record(stream)
            graphs["one_launch"].replay()
            es[1].record(stream)
            torch.cuda.synchronize()
            return es[0].elapsed_time(es[1])
        tot = 0.0
        q.qoq_set_linear_in_kernel_quant(True)
        try:
            for j, c in enumerate(cases):
                flush.zero_()
                ev[j][0].record(stream)
                q.qoq_w4a8_linear(c["X"], c["packed"], X8=c["X8"], s_x=c["s_x"], Y=c["Y"], workspace=c["ws"],
                                  stream=stream)
                ev[j][1].record(stream)
            torch.cuda.synchronize()
        finally:
            q.qoq_set_linear_in_kernel_quant(False)
        for j in range(n_sh):
            tot += ev[j][0].elapsed_time(ev[j][1])
        return tot

    def gemm_only():
        """The GEMM kernel alone, the same way (roofline of the dominant kernel)."""
        if chained:
            es[2].record(stream)
            if "gemm" in graphs:
                graphs["gemm"].replay()
            else:
                enqueue_step(stream, quant=False)
            es[3].record(stream)
            torch.cuda.synchronize()
            return es[2].elapsed_time(es[3])
        tot = 0.0
        for j, c in enumerate(cases):
            flush.zero_()
            ev[j][2].record(stream)
            q.qoq_w4a8_gemm(c["X8"], c["s_x"], c["packed"], Y=c["Y"], workspace=c["ws"], stream=stream)
            ev[j][3].record(stream)
        torch.cuda.synchronize()
        for j in range(n_sh):
            tot += ev[j][2].elapsed_time(ev[j][3])
        return tot

    def isolated(reps=3):
        """Per shape, L2 flushed, kernel(s) alone: the per-point breakdown."""
        out = []
        for j, c in enumerate(cases):
            st = gm = 0.0
            for _ in range(reps):
                flush.zero_()
                ev[j][0].record(stream)
                q.qoq_w4a8_linear(c["X"], c["packed"], X8=c["X8"], s_x=c["s_x"], Y=c["Y"], workspace=c["ws"],
                                  stream=stream)
                ev[j][1].record(stream)
                flush.zero_()
                ev[j][2].record(stream)
                q.qoq_w4a8_gemm(c["X8"], c["s_x"], c["packed"], Y=c["Y"], workspace=c["ws"], stream=stream)
                ev[j][3].record(stream)
                torch.cuda.synchronize()
                st += ev[j][0].elapsed_time(ev[j][1])
                gm += ev[j][2].elapsed_time(ev[j][3])
            out.append((st / reps, gm / reps))
        return out

    for _ in range(max(3, args.warmup)):
        one_step()
        gemm_only()
    torch.cuda.synchronize()
    if q.qoq_device_error() != q.QOQ_OK:
        raise RuntimeError("device error during warm-up")
    # Decode-sized steps are launch-bound when every kernel is launched from
    # Python; a serving loop replays them as one CUDA graph, and so does the
    # timed region (the eager step time is reported beside it).
    eager_ms = None
    if chained and not args.eager:
        eager_ms = statistics.median(one_step(eager=True) for _ in range(max(3, args.warmup)))
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        for name, kw in (("step", {}), ("gemm", {"quant": False}), ("one_launch", {})):
            g = torch.cuda.CUDAGraph()
            q.qoq_set_linear_in_kernel_quant(name == "one_launch")
            try:
                with torch.cuda.graph(g, stream=cap):
                    enqueue_step(cap, **kw)
            finally:
                q.qoq_set_linear_in_kernel_quant(False)
            graphs[name] = g
        stream.wait_stream(cap)
        for _ in range(max(3, args.warmup)):
            one_step()
            gemm_only()
        torch.cuda.synchronize()
        if q.qoq_device_error() != q.QOQ_OK:
            raise RuntimeError("device error while warming up the CUDA graphs")

    step_ms = []
    with ClockSampler(local) as clk:
        barrier(dist)
        torch.cuda.synchronize()
        t_wall = time.perf_counter()
        for _ in range(args.steps):
            step_ms.append(one_step())
        torch.cuda.synchronize()
        barrier(dist)
        wall = time.perf_counter() - t_wall
    clocks = clk.summary()
    g_ms_total = sum(gemm_only() for _ in range(args.steps)) / args.steps
    one_ms = statistics.median(one_launch_step() for _ in range(args.steps)) if (graphs or not chained) else None
    iso = isolated()
    if q.qoq_device_error() != q.QOQ_OK:
        raise RuntimeError("device error in the timed region")

    per = []
    tot_ops = g_bytes = 0.0
    for j, c in enumerate(cases):
        s = c["s"]
        pair_ms, gm_ms = iso[j]
        ops = roofline.ops(s.M, s.N, s.K)
        byt = roofline.algorithmic_bytes(s.M, s.N, s.K, s.G)
        roof = roofline.roofline_ops_per_s(s.M, s.N, s.K, s.G, peaks["int8_tops"] * 1e12, peaks["hbm_gbs"] * 1e9)
        tops = ops / (gm_ms * 1e-3) / 1e12
        per.append({"shape": s.name, "M": s.M, "K": s.K, "N": s.N, "G": s.G,
                    "isolated_step_us": round(pair_ms * 1e3, 2), "isolated_gemm_us": round(gm_ms * 1e3, 2),
                    "isolated_gemm_tops": round(tops, 2), "isolated_gemm_gbs": round(byt / (gm_ms * 1e-3) / 1e9, 1),
                    "roofline_tops": round(roof / 1e12, 2), "isolated_frac": round(tops * 1e12 / roof, 4),
                    "bound": roofline.bound(s.M, s.N, s.K, s.G, peaks["int8_tops"] * 1e12,
                                            peaks["hbm_gbs"] * 1e9)})
        tot_ops += ops
        g_bytes += byt
    tot_ms = statistics.median(step_ms)
    ms_step, value = aggregate(tot_ops, tot_ms, world, dist)
    g_ms = g_ms_total
    # roofline of the dominant kernel (the GEMM), averaged per launch
    n_hbm = sum(1 for p in per if p["bound"] == "hbm")
    bound = "hbm" if n_hbm * 2 >= len(per) else "tensor"
    if bound == "hbm":
        achieved = g_bytes / (g_ms * 1e-3) / 1e9
        rl = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
              "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None}
    else:
        achieved = sum(roofline.ops(p["M"], p["N"], p["K"]) for p in per) / (g_ms * 1e-3) / 1e12
        rl = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peaks["int8_tops"], 1),
              "unit": "TOPS", "frac": round(achieved / peaks["int8_tops"], 4), "traffic": None}
    rl["peak_source"] = peaks["source"] + (" (HBM copy)" if bound == "hbm" else " (bf16 cuBLAS x2, burst)")
    rl["kernel"] = "w4a8_gemm_kernel"
    rl["algorithmic_bytes_per_launch"] = int(g_bytes / n_sh)
    prof = os.path.join(ROOT, "profiles", f"traffic_{args.workload}.json")
    if os.path.exists(prof):
        try:
            t = json.load(open(prof))
            if t.get("kernel_source_hash") == gemm_source_hash():
                rl["traffic"] = t.get("dram_bytes_per_gemm_launch")
                rl["traffic_capture"] = t.get("capture")
        except (OSError, ValueError):
            pass

    # end to end through the public API from pinned host memory
    e2e = None
    if not args.no_e2e:
        layer_like = []
        for c in cases:
            lay = q.W4A8Linear.__new__(q.W4A8Linear)
            lay.packed = c["packed"]
            layer_like.append(lay)
        e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_sh)]
        h2d = sum(c["Xh"].numel() * 2 for c in cases)
        d2h = sum(c["Yh"].numel() * 2 for c in cases)
        tot = 0.0
        for it in range(args.warmup + args.steps):
            for j, c in enumerate(cases):
                flush.zero_()
                e2e_ev[j][0].record(stream)
                q.w4a8_linear_host(c["Xh"], layer_like[j], y_host=c["Yh"], stream=stream)
                e2e_ev[j][1].record(stream)
            torch.cuda.synchronize()
            if it >= args.warmup:
                tot += sum(e2e_ev[j][0].elapsed_time(e2e_ev[j][1]) for j in range(n_sh))
        e2e_ms = max_over_ranks(tot / args.steps, dist)
        e2e = {"value": round(world * tot_ops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TOPS",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms, 4)}

    out = {
        "metric": "W4A8 GEMM TOPS (act-quant + GEMM) and % of roofline vs batch M",
        "value": round(value, 3), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 5),
        "wall_ms_per_step": round(wall / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s8xs8->s32 (u4 weights), fp16 out", "data": "synthetic",
        "config": {"workload": work.name, "shapes": [p["shape"] for p in per],
                   "l2": ("inputs larger than L2: %d MB of distinct packed weights per step, no flush" % (wbytes >> 20))
                         if chained else "flushed before every shape (256 MB write), flush excluded from timing",
                   "timing": ("median step of %d; GEMM-only roofline from the same %s runs" %
                              (args.steps, "back-to-back" if chained else "flushed")),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": ("cuda_graph (one graph per step, programmatic dependent launch between kernels)"
                              if graphs else "eager (every kernel launched from Python)"),
                   "eager_ms_per_step": None if eager_ms is None else round(eager_ms, 5),
                   "kernels": ("per shape qoq_w4a8_linear: the per-token quantizer kernel, then the GEMM kernel "
                               "(programmatic dependent launch)"),
                   "one_launch_ms_per_step": None if one_ms is None else round(one_ms, 5)},
        "roofline": rl, "points": per, "clocks": clocks, "e2e": e2e,
        "gpu_launches": 2 * n_sh * args.steps,
        "a_operand": "smem" if args.a_smem else "tmem",
    }
    return out, cases


# ------------------------------------------------------------ CPU oracle --
def oracle_sample(work, budget_s, indices=None):
    """Time the oracle's act quant + INT32 GEMM + epilogue on the shapes of
    the workload (all, or those at `indices`), restricted to a channel
    sample sized for `budget_s` CPU seconds in total; returns (TOPS, threads,
    description)."""
    import oracle

    idx = list(range(len(work.shapes))) if indices is None else list(indices)
    n_sh = len(idx)
    per_shape = budget_s / n_sh
    tot_ops = tot_s = 0.0
    descr = []
    for i in idx:
        s = work.shapes[i]
        X, W = wl.make_case(work, i)
        Xn = X.numpy()
        rows = min(s.M, 256)
        # calibrate on 128 channels, then size the sample to the budget
        n_try = 128
        wq = oracle.quantize_weights(W[:n_try].numpy(), s.G)
        W8 = oracle.dequant_weights(wq["q"], wq["s_g"], wq["zs"], s.G)
        t0 = time.perf_counter()
        X8, s_x = oracle.quant_act(Xn[:rows])
        acc = oracle.gemm_i32(X8, W8)
        oracle.epilogue(acc, s_x, wq["s_c"])
        dt = time.perf_counter() - t0
        n_s = int(min(s.N, max(128, n_try * per_shape / max(dt, 1e-4))) // 128 * 128)
        wq = oracle.quantize_weights(W[:n_s].numpy(), s.G)
        W8 = oracle.dequant_weights(wq["q"], wq["s_g"], wq["zs"], s.G)
        t0 = time.perf_counter()
        X8, s_x = oracle.quant_act(Xn[:rows])
        acc = oracle.gemm_i32(X8, W8)
        oracle.epilogue(acc, s_x, wq["s_c"])
        dt = time.perf_counter() - t0
        tot_ops += 2.0 * rows * n_s * s.K
        tot_s += dt
        descr.append(f"{s.name}: {rows} tokens x {n_s} of {s.N} channels")
    return tot_ops / tot_s / 1e12, oracle.num_threads(), "; ".join(descr)


def oracle_single_core(work, budget_s):
    """The same oracle timing on one host core, for the workload's smallest
    shape (by operations)."""
    import oracle

    i = min(range(len(work.shapes)), key=lambda j: work.shapes[j].M * work.shapes[j].N * work.shapes[j].K)
    before = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        v, threads, descr = oracle_sample(work, budget_s, indices=[i])
    finally:
        oracle.set_num_threads(before)
    return {"value": round(v, 6), "unit": "TOPS", "cores": threads, "sample": descr}


def run_reference(args, rank, world, local, dist):
    """Reference arm: the CPU oracle, as it stands, on a bounded sample."""
    import oracle

    oracle.build()
    work = select(args)
    steps = args.steps
    budget = max(1.0, args.cpu_seconds / max(1, steps))
    vals = []
    descr = ""
    threads = oracle.num_threads()
    for _ in range(min(args.warmup, 1)):
        oracle_sample(work, budget)
    for _ in range(steps):
        v, threads, descr = oracle_sample(work, budget)
        vals.append(v)
    value = statistics.median(vals)
    return {
        "impl": "reference",
        "metric": "W4A8 GEMM TOPS (act-quant + GEMM) and % of roofline vs batch M",
        "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s8xs8->s32 (u4 weights), fp16 out", "data": "synthetic",
        "config": {"workload": work.name, "shapes": [s.name for s in work.shapes],
                   "parallelism": "host cores (oracle)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": threads, "kind": "oracle",
                         "sample": descr},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, 0, int(os.environ.get("WORLD_SIZE", "1")), 0, None)), flush=True)
        return 0
    rank, world, local, dist = dist_setup(args.gpus)
    try:
        out, cases = run_ours(args, rank, world, local, dist)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, threads, descr = oracle_sample(select(args), args.cpu_seconds)
            try:
                single = oracle_single_core(select(args), min(5.0, args.cpu_seconds))
            except Exception as e:  # a side figure: report why, keep the line
                single = {"error": f"{type(e).__name__}: {e}"}
            out["cpu_baseline"] = {"value": round(v, 6), "unit": "TOPS", "cores": threads, "kind": "oracle",
                                   "sample": descr, "single_core": single}
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
