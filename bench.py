"""Benchmark of the W4A8 linear layer on B200: TOPS and % of roofline vs M.

One step = one pass of the whole hot path -- per-token activation
quantization, then the W4A8 GEMM with its epilogue -- over every shape of the
workload, with weights packed offline (untimed) and resident in HBM.

The default workload is the batch-size sweep the metric is quoted on:
M = 1, 2, 4, ..., 8192 tokens on K = N = 8192 with g128 weights (14 GEMMs
per step, 485 MB of distinct packed weights).  `--workload
decode|large_batch|qwen|tiny` selects the other workloads for ad-hoc
measurement.

Timing: when the distinct packed weights of a step exceed 1.5x L2
(126 MB), the shapes run back to back, replayed from one CUDA graph, and the
step is bracketed by CUDA events on the launching stream: every weight byte
comes from HBM, because the step has cycled more than L2 since it last read
the same weights.  Smaller workloads flush L2 (a 256 MB write) before every
shape instead, bracket each shape with events (flush excluded) and sum.
K timed steps follow W untimed ones, bracketed by a barrier and a device
synchronize; with N > 1 every rank runs the same workload (replicas, weak
scaling) and the time is the max over ranks.

The roofline of the dominant kernel (the GEMM) is reported per regime: the
HBM-bound shapes and the tensor-bound shapes each run as their own chain of
GEMM launches (again one graph, weights from HBM), and `achieved` is their
algorithmic bytes (or operations) over that chain's time.  Per shape, an
isolated run (L2 flushed, the kernels alone) gives the per-point breakdown.

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
GEMM_SOURCES = ("qoq_gemm.cu", "qoq_epilogue.cuh", "qoq_layout.cuh", "qoq_ptx.cuh", "qoq_internal.h", "qoq_quant.cuh")


def code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed, for
    hashing: a change of wording leaves the hash as it was."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="sweep", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--only", default=None,
                    help="restrict the workload to one shape name (for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-kv4", action="store_true",
                    help="skip the KV4 decode-attention measurement reported beside the GEMM")
    ap.add_argument("--no-w8a8", action="store_true",
                    help="skip the W8A8 yardstick (the same kernel with INT8 weights) beside each point")
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
                 "--format=csv,noheader,nounits", "-lms", "50"],
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


# ----------------------------------------------------- KV4 attention leg --
KV4_SHAPES = (  # (name, sequences, query heads, KV heads, cached tokens); head dimension 128
    ("llama3_8b_gqa4_B32_L4096", 32, 32, 8, 4096),
    ("qwen15_72b_mha_B8_L4096", 8, 64, 64, 4096),
)


def run_kv4(dev, peaks, flush, reps=20):
    """KV4 decode attention over a synthetic 4-bit cache: device time of the
    two kernels (chunks + combine) per call, L2 flushed before each call,
    against the HBM roofline of its algorithmic bytes (the 4-bit codes of K
    and V, their per-channel factors, the query and the output)."""
    import w4a8_integer_gemm_b200 as q
    out = []
    stream = torch.cuda.current_stream()
    for name, B, Hq, Hkv, L in KV4_SHAPES:
        d = 128
        K, V = wl.make_kv(B, Hkv, L, d, seed=7 + L)
        Q = wl.make_queries(B, Hq, d, seed=8 + L).to(dev)
        cache = q.qoq_kv4_cache_quantize(K.to(dev), V.to(dev))
        del K, V
        ws = torch.empty(q.qoq_kv4_attention_workspace_bytes(B, Hq, Hkv, L, d), dtype=torch.uint8, device=dev)
        o = torch.empty(B, Hq, d, dtype=torch.float16, device=dev)
        for _ in range(3):
            q.qoq_kv4_decode_attention(Q, cache, out=o, workspace=ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0.record(stream)
            q.qoq_kv4_decode_attention(Q, cache, out=o, workspace=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        byt = B * Hkv * L * d + 3 * B * Hkv * d * 2 + 2 * B * Hq * d * 2
        gbs = byt / (ms * 1e-3) / 1e9
        # ALU floor: the products run on the tensor cores; expanding the
        # 4-bit codes into FP16 operands takes about 1.5 instructions per
        # code (K and V), 128 lanes per SM per clock at the maximum SM clock
        alu_ops = 1.5 * 2 * B * Hkv * L * d
        alu_rate = 148 * 128 * peaks.get("sm_max_mhz", 1965.0) * 1e6
        out.append({"shape": name, "B": B, "Hq": Hq, "Hkv": Hkv, "L": L, "d": d, "us": round(ms * 1e3, 2),
                    "algorithmic_bytes": byt, "achieved_gbs": round(gbs, 1),
                    "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                    "code_expansion_floor_us": round(alu_ops / alu_rate * 1e6, 2),
                    "bound": "hbm" if byt / (peaks["hbm_gbs"] * 1e9) >= alu_ops / alu_rate else "alu"})
        del cache, ws
    torch.cuda.synchronize()
    if q.qoq_device_error() != q.QOQ_OK:
        raise RuntimeError("device error in the KV4 attention leg")
    return {"kernels": "kv4_attn_kernel + kv4_combine_kernel", "timing": "isolated, L2 flushed, median of %d" % reps,
            "points": out}


# --------------------------------------------------------------- our arm --
def load_traffic(workload_name: str, path: str = None):
    """The ncu DRAM-traffic record of this workload's GEMM, if its kernel
    source hash still matches the current code: {capture shape name:
    {...}} or {} (the counters describe that kernel and no later one)."""
    prof = path or os.path.join(ROOT, "profiles", f"traffic_{workload_name}.json")
    try:
        with open(prof) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return {}
    if t.get("kernel_source_hash") != gemm_source_hash():
        return {}
    return t.get("captures", {})


def regime_roofline(bound, shapes, ms, peaks, traffic, sm_mhz=None):
    """Roofline record of the GEMM over a chain of shapes of one regime
    (all HBM-bound or all tensor-bound), timed back to back: `ms` is the
    chain's time.  `traffic` comes from one ncu capture of a representative
    shape of the regime, with that shape's algorithmic bytes beside it.
    `sm_mhz`: the median SM clock seen under load (the maximum, 1965 MHz,
    when no clock was sampled), for the MMA issue ceiling of the tensor
    regime."""
    n = len(shapes)
    byt = sum(roofline.algorithmic_bytes(x.M, x.N, x.K, x.G) for x in shapes)
    ops = sum(roofline.ops(x.M, x.N, x.K) for x in shapes)
    if bound == "hbm":
        achieved = byt / (ms * 1e-3) / 1e9
        rl = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
              "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
              "peak_source": peaks["source"] + " (HBM copy)"}
    else:
        achieved = ops / (ms * 1e-3) / 1e12
        rl = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peaks["int8_tops"], 1),
              "unit": "TOPS", "frac": round(achieved / peaks["int8_tops"], 4), "traffic": None,
              "peak_source": peaks["source"] + " (2 x bf16 cuBLAS burst)",
              "frac_of_sustained_peak": round(achieved / peaks["int8_tops_sustained"], 4)}
        ceil = roofline.mma_issue_ceiling_tops(float(sm_mhz) if sm_mhz else 1965.0)
        rl["mma_issue_ceiling_tops"] = round(ceil, 1)
        rl["frac_of_mma_issue_ceiling"] = round(achieved / ceil, 4)
    small = [x.name for x in shapes if x.M <= 8]
    kern = "w4a8_gemm_kernel" + (f" (w4a8_gemv_kernel for {', '.join(small)})" if small else "")
    rl.update({"kernel": kern, "launches": n, "chain_us": round(ms * 1e3, 2),
               "us_per_launch": round(ms * 1e3 / n, 3), "shapes": [x.name for x in shapes],
               "algorithmic_bytes_per_launch": int(byt / n), "ops_per_launch": int(ops / n)})
    rep = [k for k in traffic if k in {x.name for x in shapes}]
    if rep:
        t = traffic[rep[0]]
        rl["traffic"] = t["dram_bytes"]
        rl["traffic_shape"] = rep[0]
        rl["traffic_algorithmic_bytes"] = t["algorithmic_bytes"]
        rl["traffic_capture"] = t.get("capture")
        if t.get("tensor_pipe_pct") is not None:
            rl["ncu_tensor_pipe_pct"] = t["tensor_pipe_pct"]
    return rl


def run_ours(args, rank, world, local, dist):
    import w4a8_integer_gemm_b200 as q

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q.lib()
    q.qoq_set_gemm_a_in_tmem(not args.a_smem)
    peaks = roofline.load_peaks()
    P8, BW = peaks["int8_tops"] * 1e12, peaks["hbm_gbs"] * 1e9
    work = select(args)
    stream = torch.cuda.current_stream()

    # inputs: seeded synthetic draws, packed offline, resident in HBM
    cases = []
    for i, s in enumerate(work.shapes):
        X, W = wl.make_case(work, i)
        Wd = W.to(dev)
        packed = q.qoq_pack_weights(Wd, s.G)
        w8 = None if args.no_w8a8 else q.qoq_quantize_weights_w8(Wd)
        del Wd
        Xd = X.to(dev)
        X8 = torch.empty(s.M, s.K, dtype=torch.int8, device=dev)
        s_x = torch.empty(max(s.M, 8), dtype=torch.int16, device=dev)
        Y = torch.empty(s.M, s.N, dtype=torch.float16, device=dev)
        ws = torch.zeros(q.qoq_gemm_workspace_bytes(s.M, s.N, s.K, s.G), dtype=torch.uint8, device=dev)
        Xh = X.pin_memory()
        Yh = torch.empty(s.M, s.N, dtype=torch.float16, pin_memory=True)
        cases.append(dict(s=s, packed=packed, w8=w8, X=Xd, X8=X8, s_x=s_x, Y=Y, ws=ws, Xh=Xh, Yh=Yh,
                          bound=roofline.bound(s.M, s.N, s.K, s.G, P8, BW)))
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
    # the GEMM's regimes, each chained on its own when its weights alone
    # exceed the L2 the same way
    regimes = {}
    for b in ("hbm", "tensor"):
        sub = [c for c in cases if c["bound"] == b]
        if sub:
            regimes[b] = sub
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [[E() for _ in range(4)] for _ in range(n_sh)]
    es = [E(), E()]

    def enqueue(st, subset, layer=True):
        """Launch on stream st, per shape of `subset`, the layer call
        (qoq_w4a8_linear: the quantizer kernel, then the GEMM kernel), the
        GEMM kernel alone, or (layer="w8a8") the W8A8 yardstick's GEMM."""
        for c in subset:
            if layer == "w8a8":
                q.qoq_w8a8_gemm(c["X8"], c["s_x"], c["w8"][0], c["w8"][1], Y=c["Y"], workspace=c["ws"], stream=st)
            elif layer:
                q.qoq_w4a8_linear(c["X"], c["packed"], X8=c["X8"], s_x=c["s_x"], Y=c["Y"], workspace=c["ws"],
                                  stream=st)
            else:
                q.qoq_w4a8_gemm(c["X8"], c["s_x"], c["packed"], Y=c["Y"], workspace=c["ws"], stream=st)

    graphs = {}

    def timed(name, subset, layer=True, eager=False):
        """Device time in ms of one pass over `subset`: back to back from a
        graph when chained, else per shape after an L2 flush (summed)."""
        if chained:
            es[0].record(stream)
            if name in graphs and not eager:
                graphs[name].replay()
            else:
                enqueue(stream, subset, layer)
            es[1].record(stream)
            torch.cuda.synchronize()
            return es[0].elapsed_time(es[1])
        tot = 0.0
        for c in subset:
            j = cases.index(c)
            flush.zero_()
            ev[j][0].record(stream)
            enqueue(stream, [c], layer)
            ev[j][1].record(stream)
            torch.cuda.synchronize()
            tot += ev[j][0].elapsed_time(ev[j][1])
        return tot

    def isolated(reps=3):
        """Per shape, L2 flushed, kernel(s) alone: the per-point breakdown
        (layer call, GEMM, and the W8A8 yardstick's GEMM)."""
        out = []
        for j, c in enumerate(cases):
            st = gm = w8 = 0.0
            for _ in range(reps):
                if c["w8"] is not None:
                    flush.zero_()
                    ev[j][0].record(stream)
                    enqueue(stream, [c], "w8a8")
                    ev[j][1].record(stream)
                    torch.cuda.synchronize()
                    w8 += ev[j][0].elapsed_time(ev[j][1])
                flush.zero_()
                ev[j][0].record(stream)
                enqueue(stream, [c], True)
                ev[j][1].record(stream)
                flush.zero_()
                ev[j][2].record(stream)
                enqueue(stream, [c], False)
                ev[j][3].record(stream)
                torch.cuda.synchronize()
                st += ev[j][0].elapsed_time(ev[j][1])
                gm += ev[j][2].elapsed_time(ev[j][3])
            out.append((st / reps, gm / reps, w8 / reps if c["w8"] is not None else None))
        return out

    chains = {"step": (cases, True)}
    for b, sub in regimes.items():
        chains["gemm_" + b] = (sub, False)
        if not args.no_w8a8:
            chains["w8a8_" + b] = (sub, "w8a8")
    for _ in range(max(3, args.warmup)):
        for name, (sub, layer) in chains.items():
            timed(name, sub, layer)
    torch.cuda.synchronize()
    if q.qoq_device_error() != q.QOQ_OK:
        raise RuntimeError("device error during warm-up")
    # A serving loop replays a step's launches as one CUDA graph, and so does
    # the timed region (the eager step time is reported beside it).
    eager_ms = None
    if chained and not args.eager:
        eager_ms = statistics.median(timed("step", cases, True, eager=True) for _ in range(max(3, args.warmup)))
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        for name, (sub, layer) in chains.items():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                enqueue(cap, sub, layer)
            graphs[name] = g
        stream.wait_stream(cap)
        for _ in range(max(3, args.warmup)):
            for name, (sub, layer) in chains.items():
                timed(name, sub, layer)
        torch.cuda.synchronize()
        if q.qoq_device_error() != q.QOQ_OK:
            raise RuntimeError("device error while warming up the CUDA graphs")

    step_ms = []
    with ClockSampler(local) as clk:
        barrier(dist)
        torch.cuda.synchronize()
        t_wall = time.perf_counter()
        for _ in range(args.steps):
            step_ms.append(timed("step", cases, True))
        torch.cuda.synchronize()
        barrier(dist)
        wall = time.perf_counter() - t_wall
    clocks = clk.summary()
    chain_ms = {b: statistics.median(timed("gemm_" + b, sub, False) for _ in range(args.steps))
                for b, sub in regimes.items()}
    w8_chain_ms = {} if args.no_w8a8 else {
        b: statistics.median(timed("w8a8_" + b, sub, "w8a8") for _ in range(args.steps)) for b, sub in regimes.items()}
    iso = isolated()
    if q.qoq_device_error() != q.QOQ_OK:
        raise RuntimeError("device error in the timed region")

    per = []
    tot_ops = 0.0
    for j, c in enumerate(cases):
        s = c["s"]
        pair_ms, gm_ms, w8_ms = iso[j]
        ops = roofline.ops(s.M, s.N, s.K)
        byt = roofline.algorithmic_bytes(s.M, s.N, s.K, s.G)
        roof = roofline.roofline_ops_per_s(s.M, s.N, s.K, s.G, P8, BW)
        tops = ops / (gm_ms * 1e-3) / 1e12
        per.append({"shape": s.name, "M": s.M, "K": s.K, "N": s.N, "G": s.G, "bound": c["bound"],
                    "isolated_step_us": round(pair_ms * 1e3, 2), "isolated_gemm_us": round(gm_ms * 1e3, 2),
                    "isolated_gemm_tops": round(tops, 2), "isolated_gemm_gbs": round(byt / (gm_ms * 1e-3) / 1e9, 1),
                    "roofline_tops": round(roof / 1e12, 2), "isolated_frac": round(tops * 1e12 / roof, 4)})
        if w8_ms is not None:
            b8 = roofline.algorithmic_bytes_w8(s.M, s.N, s.K)
            roof8 = min(P8, ops * BW / b8)
            per[-1].update({"w8a8_isolated_gemm_us": round(w8_ms * 1e3, 2),
                            "w8a8_isolated_gemm_tops": round(ops / (w8_ms * 1e-3) / 1e12, 2),
                            "w8a8_roofline_tops": round(roof8 / 1e12, 2),
                            "w8a8_isolated_frac": round(ops / (w8_ms * 1e-3) / roof8, 4),
                            "w4a8_speedup_over_w8a8": round(w8_ms / gm_ms, 3)})
        tot_ops += ops
    tot_ms = statistics.median(step_ms)
    ms_step, value = aggregate(tot_ops, tot_ms, world, dist)
    traffic = load_traffic(args.workload)
    by_bound = {b: regime_roofline(b, [c["s"] for c in sub], chain_ms[b], peaks, traffic, clocks.get("sm_mhz"))
                for b, sub in regimes.items()}
    # the dominant kernel's regime: where the GEMM spends most of the step
    dom = max(by_bound, key=lambda b: by_bound[b]["chain_us"])
    rl = dict(by_bound[dom])
    rl["by_bound"] = by_bound
    # the W8A8 yardstick over the same chains (its own algorithmic bytes:
    # INT8 weights, N*K), and where it overtakes W4A8 (isolated points)
    w8a8 = None
    if w8_chain_ms:
        w8a8 = {"kernel": "w4a8_gemm_kernel (W8 variant: INT8 weights by TMA, no dequantization)", "by_bound": {}}
        for b, sub in regimes.items():
            shp = [c["s"] for c in sub]
            ms = w8_chain_ms[b]
            ops_b = sum(roofline.ops(x.M, x.N, x.K) for x in shp)
            byt_b = sum(roofline.algorithmic_bytes_w8(x.M, x.N, x.K) for x in shp)
            ent = {"chain_us": round(ms * 1e3, 2), "tops": round(ops_b / (ms * 1e-3) / 1e12, 1),
                   "w4a8_chain_us": round(chain_ms[b] * 1e3, 2),
                   "w4a8_speedup": round(ms / chain_ms[b], 3)}
            if b == "hbm":
                ach = byt_b / (ms * 1e-3) / 1e9
                ent.update({"achieved_gbs": round(ach, 1), "frac_of_hbm": round(ach / peaks["hbm_gbs"], 4)})
            else:
                ach = ops_b / (ms * 1e-3) / 1e12
                ent.update({"frac_of_int8_peak": round(ach / peaks["int8_tops"], 4)})
            w8a8["by_bound"][b] = ent
        cross = [p["M"] for p in per if "w4a8_speedup_over_w8a8" in p and p["w4a8_speedup_over_w8a8"] < 1.0]
        w8a8["first_M_where_w8a8_is_faster"] = min(cross) if cross else None
        # the pages' roofline argument ("QServe: Low Bit Width Does Not
        # Guarantee High Throughput", section 2, Figure 3) redone with this
        # GPU's measured peaks: per weight element, W4A16 moves 0.5 byte at
        # the FP16 peak (half the INT8 peak), W8A8 1 byte at the INT8 peak,
        # W4A8 0.5 byte at the INT8 peak
        w4a16, w8, w4 = (P8 / 2, 0.5), (P8, 1.0), (P8, 0.5)
        w8a8["roofline_model_crossovers_m"] = {
            "w4a16_vs_w8a8": roofline.crossover_m(w4a16, w8, BW),
            "w4a8_vs_w8a8_equal_from": roofline.crossover_m(w4, w8, BW)}

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
        # one call per shape, each synchronized before the next
        tot = 0.0
        for it in range(max(3, args.warmup) + args.steps):
            for j, c in enumerate(cases):
                flush.zero_()
                e2e_ev[j][0].record(stream)
                q.w4a8_linear_host(c["Xh"], layer_like[j], y_host=c["Yh"], stream=stream)
                e2e_ev[j][1].record(stream)
            torch.cuda.synchronize()
            if it >= max(3, args.warmup):
                tot += sum(e2e_ev[j][0].elapsed_time(e2e_ev[j][1]) for j in range(n_sh))
        serial_ms = max_over_ranks(tot / args.steps, dist)
        # the step's calls pipelined: copies of one shape overlap the kernels
        # of the others
        calls = [(c["Xh"], layer_like[j], c["Yh"]) for j, c in enumerate(cases)]
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for it in range(max(3, args.warmup) + args.steps):
            p0.record(stream)
            q.w4a8_linear_host_many(calls, stream=stream)
            p1.record(stream)
            torch.cuda.synchronize()
            if it >= max(3, args.warmup):
                tot += p0.elapsed_time(p1)
        e2e_ms = max_over_ranks(tot / args.steps, dist)
        e2e = {"value": round(world * tot_ops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TOPS",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms, 4),
               "call": "w4a8_linear_host_many over the step's shapes, cut into row blocks of about 16 MB: "
                       "X pinned host -> device, layer call, Y -> pinned host on three streams chained by "
                       "events, one synchronize at the end",
               "serial": {"value": round(world * tot_ops / (serial_ms * 1e-3) / 1e12, 3), "ms_per_step":
                          round(serial_ms, 4), "call": "w4a8_linear_host per shape, each synchronized"}}

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
                   "timing": ("median step of %d; GEMM roofline per regime from chains of the same %s runs" %
                              (args.steps, "back-to-back" if chained else "flushed")),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": ("cuda_graph (one graph per step, programmatic dependent launch between kernels)"
                              if graphs else "eager (every kernel launched from Python)"),
                   "eager_ms_per_step": None if eager_ms is None else round(eager_ms, 5),
                   "kernels": ("per shape qoq_w4a8_linear: the per-token quantizer kernel, then the GEMM kernel "
                               "(programmatic dependent launch)")},
        "roofline": rl, "points": per, "clocks": clocks, "e2e": e2e, "w8a8_yardstick": w8a8,
        "kv4_attention": None if args.no_kv4 else run_kv4(dev, dict(peaks, sm_max_mhz=clocks.get("sm_max_mhz") or 1965.0),
                                                          flush),
        "gpu_launches": 2 * n_sh * args.steps,
        "a_operand": "smem" if args.a_smem else "tmem",
    }
    return out, cases


# ------------------------------------------------------------ CPU oracle --
def oracle_sample(work, cpu_s, indices=None):
    """Time the oracle's act quant + INT32 GEMM + epilogue on the shapes of
    the workload (all, or those at `indices`), restricted to a channel
    sample sized for `cpu_s` CPU seconds in total; returns (TOPS, threads,
    description)."""
    import oracle

    idx = list(range(len(work.shapes))) if indices is None else list(indices)
    n_sh = len(idx)
    per_shape = cpu_s / n_sh
    tot_ops = tot_s = 0.0
    descr = []
    for i in idx:
        s = work.shapes[i]
        X, W = wl.make_case(work, i)
        Xn = X.numpy()
        rows = min(s.M, 256)
        # calibrate on 128 channels, then size the sample to that time
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


def oracle_single_core(work, cpu_s):
    """The same oracle timing on one host core, for the workload's smallest
    shape (by operations)."""
    import oracle

    i = min(range(len(work.shapes)), key=lambda j: work.shapes[j].M * work.shapes[j].N * work.shapes[j].K)
    before = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        v, threads, descr = oracle_sample(work, cpu_s, indices=[i])
    finally:
        oracle.set_num_threads(before)
    return {"value": round(v, 6), "unit": "TOPS", "cores": threads, "sample": descr}


def run_reference(args, rank, world, local, dist):
    """Reference arm: the CPU oracle, as it stands, on a bounded sample."""
    import oracle

    oracle.build()
    work = select(args)
    steps = args.steps
    per_step_s = max(1.0, args.cpu_seconds / max(1, steps))
    vals = []
    descr = ""
    threads = oracle.num_threads()
    for _ in range(min(args.warmup, 1)):
        oracle_sample(work, per_step_s)
    for _ in range(steps):
        v, threads, descr = oracle_sample(work, per_step_s)
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
