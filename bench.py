"""Benchmark of the CSA / HCA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Headline workload: CSA decode at 64K context (16 sequences, FP8 indexer,
top-k 512, window 128, 64 heads x 512).  A step is one fused decode step for
the whole batch (compress the entry the new token completes, quantise the
index query, score every entry, select top-k, attend over selection + window)
with inputs resident in HBM.  L2 is flushed (a 256 MiB write) before every
timed step, outside the step's CUDA events.  The K-step timed region (each
bracketed by a barrier and a device synchronise) is repeated until the whole
run spans at least a second, so the clock sampler sees the GPU under load; the
line reports the repeat count and the median repeat.  Multi-GPU runs are
independent replicas (the path has no exchange step): value = all ranks'
tokens / max over ranks of the device time.

Without --workload the same run also measures, as sub-records under "sub",
the other parts of the metric: CSA decode at 1M context (NVFP4 indexer), HCA
decode at 1M context and CSA prefill at 32K (FP8 indexer), each with its own
roofline, per-kernel fractions, clocks and oracle baseline.  The FP8 dense
tensor-core peak of the prefill roofline is measured in the same run (a plain
torch._scaled_mm at 8192^3, best of 10).

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
this host's cores on a bounded sample of the same workload instead.
"""

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_sparse_05_b200 import _lib as L  # noqa: E402
from long_context_sparse_05_b200 import runner, synth, workloads  # noqa: E402

METRIC = "CSA decode tok/s/B200 at 64K & 1M ctx; % of HBM roofline; prefill % TC peak"
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons; ``window`` keeps the samples taken
    while the timed region ran (host wall-clock bounds), widened to the nearest samples."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []   # (host time, sm, max, reasons)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
            time.sleep(0.5)
        except OSError:
            self.proc = None

    def _read(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                sm, mx = float(f[2]), float(f[3])
            except ValueError:
                continue
            rs = [nm for nm, v in zip(names, f[6:10]) if v.lower() == "active"]
            self.samples.append((time.time(), sm, mx, rs))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside and self.samples:
            # the timed region was shorter than the sampling period: nearest samples on each side
            before = [x for x in self.samples if x[0] < t0][-1:]
            after = [x for x in self.samples if x[0] > t1][:1]
            inside = before + after
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({r for x in inside for r in x[3]})
        return {"sm_mhz": float(np.median([x[1] for x in inside])), "sm_max_mhz": inside[-1][2],
                "reasons": reasons, "samples": len(inside),
                "timed_region_s": round(t1 - t0, 4)}


def dist_setup(n_gpus):
    """One process per GPU: the rank's device is made current before the process group
    exists, so that NCCL binds to it (its barriers and reductions run there)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Max of a host scalar over the ranks (NCCL ranks reduce on their GPU, gloo on the CPU)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(ms_local, tokens_local, world):
    """Whole-job throughput of independent replicas: all ranks' tokens over the slowest rank's
    device time.  Returns (ms_per_step, tokens_per_step, tokens_per_second)."""
    ms = max_over_ranks(ms_local, world)
    tokens = tokens_local * world
    return ms, tokens, tokens / (ms * 1e-3)


HOST_LEAD_CYCLES = 100_000   # device spin per timed step before the loop (~50 us at 1.9 GHz)


def timed_loop(fn, steps, flush_buf, stream, warm=0, nvtx=None):
    """Per-step CUDA events on the launching stream; L2 flushed between steps, outside the events.

    ``warm`` untimed calls go first (the first launch of a kernel also loads its
    module).  ``nvtx`` names a push/pop range around the timed calls, so a
    profiler can select exactly the timed launches.
    """
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    with torch.cuda.stream(stream):
        for _ in range(warm):
            flush_buf.zero_()
            fn()
        torch.cuda.synchronize()
        if nvtx:
            torch.cuda.nvtx.range_push(nvtx)
        # the device first spins for ~50 us per step (outside every event pair), so that the
        # host has queued each call before its start event fires: the events then time the
        # device work, not the host's Python and ctypes overhead per call
        torch.cuda._sleep(int(steps * HOST_LEAD_CYCLES))
        for a, b in evs:
            flush_buf.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        if nvtx:
            torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def timed_region(fn, steps, flush, stream, world, min_span_s, max_repeats=4000):
    """The K-step timed loop, each run bracketed by a barrier and a synchronise, repeated until
    the runs span ``min_span_s`` of wall time.  One calibration run fixes the repeat count
    (its wall time is maxed over the ranks, so every rank repeats equally often).
    Returns (mean ms per step of each repeat, host time at start, at end)."""
    barrier(world)
    torch.cuda.synchronize()
    timed_loop(fn, steps, flush, stream)   # one-time costs of the loop itself (events, first calls)
    torch.cuda.synchronize()
    c0 = time.time()
    timed_loop(fn, steps, flush, stream)
    c1 = time.time()
    one = max_over_ranks(c1 - c0, world)
    reps = int(min(max_repeats, max(1, math.ceil(min_span_s / max(one, 1e-6)))))
    out = []
    t0 = time.time()
    for r in range(reps):
        barrier(world)
        torch.cuda.synchronize()
        times = timed_loop(fn, steps, flush, stream, nvtx="timed_steps" if r == 0 else None)
        out.append(float(np.mean(times)))
        barrier(world)
    t1 = time.time()
    return out, t0, t1


# DRAM bytes (read + write) of one launch, from the ncu captures under profiles/, per unit the
# launch processes, so that the figure scales to the launch timed:
#   FP8 indexer: per key entry (ncu_full_index_scores_tc_csa_decode_64k_b4.md: batch 4,
#     16384 entries per sequence); NVFP4 indexer: per key entry
#     (ncu_full_index_scores_fp4_ctx256k_b2.md: batch 2, 65536 entries per sequence);
#   decode attention of the 64K workload: per query (ncu_full_attn_tc_csa_decode_64k_b4.md:
#     batch 4, 640 rows per query).
# The traffic is linear in those units.  A kernel changed after its capture has no entry
# here (its traffic is then reported as null).
PROFILED_TRAFFIC = {
    ("index_scores", "fp8"): ("entries", 8773376 / (4 * 16384)),
    ("index_scores", "nvfp4"): ("entries", 9498368 / (2 * 65536)),
    ("sparse_attn", "csa_decode_64k_fp8"): ("queries", 3032576 / 4),
}


def profiled_traffic(w, kernel):
    rec = PROFILED_TRAFFIC.get((kernel, w.idx_dtype)) or PROFILED_TRAFFIC.get((kernel, w.name))
    if rec is None:
        return None
    unit, per = rec
    return round(per * w.b * (w.E if unit == "entries" else 1))


def kernel_record(us, amount, peak, unit="GB/s", bound="hbm"):
    """Achieved rate of one kernel (algorithmic bytes or FLOPs per launch / its event time)."""
    scale = 1e9 if unit == "GB/s" else 1e12
    rate = amount / (us * 1e-6) / scale
    return {"us": round(us, 2), "bound": bound, "work": int(amount), "achieved": round(rate, 1),
            "unit": unit, "peak": peak, "frac": round(rate / peak, 4)}


def decode_stage_bytes(w):
    """Algorithmic bytes of each decode stage call, every input read and output written once
    (b sequences).  compress: the raw C and Z rows of the completing block (and of the previous
    block for c4a) plus the entry; quantize: q_I in, codes and scales out; index_scores: every
    key row with its scale, the query codes, scales and weights, the scores out; topk: the
    scores in, the selection out; sparse_attn: the selected and window rows, q in, out."""
    eb = 2 if w.dtype == "bf16" else 4
    rows_in = (4 if w.overlap else 2) * w.m
    d = {"compress": w.b * (rows_in * w.c * eb + w.c * eb)}
    if w.kind != "hca_decode":
        krow = {"fp8": w.c_I + 4, "nvfp4": w.c_I // 2 + w.c_I // 16, "f32": 4 * w.c_I}[w.idx_dtype]
        d["quantize"] = w.b * w.H_I * (w.c_I * eb + krow)
        d["index_scores"] = w.b * w.E * krow + w.b * w.H_I * (krow + 4) + w.b * w.E * 2
        d["topk"] = w.b * w.E * 2 + w.b * (w.k + 1) * 4
        d["sparse_attn"] = w.b * ((w.k + w.n_w) * w.c * eb + 2 * w.H * w.c * eb + w.k * 4)
    else:
        d["sparse_attn"] = w.b * ((w.E + w.n_w) * w.c * eb + 2 * w.H * w.c * eb)
    return d


def bench_decode(w, args, world, rank, peaks, min_span_s):
    dev = "cuda"
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    inp = synth.make_inputs(w, device=dev)
    st = runner.DecodeState(w, inp)
    st.build_caches()
    torch.cuda.synchronize()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    step = lambda: st.step(stream)   # noqa: E731
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    reps, t0, t1 = timed_region(step, args.steps, flush, stream, world, min_span_s)
    ck = clocks.stop(t0, t1)
    ck["repeats"] = len(reps)
    ms, tokens_per_step, value = aggregate(float(np.median(reps)), w.b, world)

    # every stage call of the step timed alone; the longest one is the roofline kernel
    stage = stage_times_decode(w, st, args.steps, flush, stream)
    sbytes = decode_stage_bytes(w)
    kernels = {k: kernel_record(stage[k] * 1e3, sbytes[k], peaks["hbm"]) for k in stage}
    dom = max(kernels, key=lambda k: kernels[k]["us"])
    roof = dict(kernels[dom])
    roof.pop("us")
    roof["kernel"] = dom
    roof["traffic"] = profiled_traffic(w, dom)
    step_bytes = runner.decode_bytes_per_step(w)

    e2e = e2e_decode(w, st, args.steps, flush, stream, world)
    del st, inp, flush
    torch.cuda.empty_cache()
    return dict(value=value, ms=ms, tokens_per_step=tokens_per_step, clocks=ck, stage=stage,
                roofline=roof, kernels=kernels,
                step_roofline={"algorithmic_bytes": step_bytes,
                               "achieved_gbs": round(step_bytes / (ms * 1e-3) / 1e9, 1),
                               "frac": round(step_bytes / (ms * 1e-3) / 1e9 / peaks["hbm"], 4)},
                e2e=e2e, launches=runner.decode_launches_per_step(w) * args.steps * len(reps),
                repeats=len(reps))


def stage_times_decode(w, st, steps, flush, stream):
    """Mean ms of each stage call of the decode step, each timed alone with events."""
    x = st.x
    E = w.E
    t = w.n - 1
    qpos = torch.full((w.b,), t, dtype=torch.int32, device="cuda")
    res = {}
    cp = runner.compress_params(w, "main")
    res["compress"] = np.mean(timed_loop(lambda: L.csa_compress(
        cp, x["C_a"], x["Z_a"], x["B_a"], x.get("C_b"), x.get("Z_b"), x.get("B_b"), w.b, w.n, E - 1,
        1, st.E_cap, st.kv_cache, None, stream), steps, flush, stream, warm=3))
    if w.kind != "hca_decode":
        codes = torch.empty((w.b * w.H_I, runner.row_bytes(w.idx_dtype, w.c_I)), dtype=torch.uint8,
                            device="cuda")
        qs = torch.empty((w.b * w.H_I,), dtype=torch.float32, device="cuda") if w.idx_dtype == "fp8" \
            else torch.empty((w.b * w.H_I, w.c_I // 16), dtype=torch.uint8, device="cuda")
        res["quantize"] = np.mean(timed_loop(lambda: L.csa_quantize(
            L.DTYPE[w.dtype], L.DTYPE[w.idx_dtype], x["q_I"], w.b * w.H_I, w.c_I, codes, qs, stream),
            steps, flush, stream, warm=3))
        scores = torch.empty((w.b, E), dtype=torch.bfloat16, device="cuda")
        ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[w.idx_dtype],
                           score_dtype=L.CSA_BF16)
        res["index_scores"] = np.mean(timed_loop(lambda: L.csa_index_scores(
            ip, codes, qs, x["w"], st.kI_cache, st.kI_scales, qpos, w.b, 1, st.E_cap, E, scores,
            stream), steps, flush, stream, warm=3))
        tkb = L.csa_topk_workspace_size(L.CSA_BF16, w.b, 1, E, w.k)
        tkws = torch.empty((max(tkb, 256),), dtype=torch.uint8, device="cuda")
        res["topk"] = np.mean(timed_loop(lambda: L.csa_topk(
            scores, L.CSA_BF16, qpos, w.m, w.b, 1, E, w.k, st.idx, st.count, tkws, tkb, stream),
            steps, flush, stream, warm=3))
        idx, cnt = st.idx, st.count
    else:
        idx = cnt = None
    ap = L.AttnParams(H=w.H, d=w.c, n_w=w.n_w, scale=w.scale, m=w.m,
                      k=0 if idx is None else w.k, dtype=L.DTYPE[w.dtype])
    wsb = L.csa_sparse_attn_workspace_size(ap, w.b, 1, st.E_cap)
    ws = torch.empty((max(wsb, 256),), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(st.out)
    res["sparse_attn"] = np.mean(timed_loop(lambda: L.csa_sparse_attn(
        ap, x["q"], st.kv_cache, st.E_cap, idx, cnt, x["C_a"], w.n, qpos, x["sink"], w.b, 1, out,
        None, ws, wsb, stream), steps, flush, stream, warm=3))
    return {k: float(v) for k, v in res.items()}


L2_BYTES = 126 * 1024 * 1024


def e2e_decode(w, st, steps, flush, stream, world=1):
    """The decode step through the public serving call, csa_decode_paged, with host inputs.

    The caches live in pages and the per-sequence state (window and raw tail rings) on
    the device, as a server keeps them; each step copies only what a new token brings
    (its raw C / Z rows of both branches, its window row, q, q_I, w and the positions)
    from one pinned host buffer to one device staging buffer (a single H2D copy), runs
    the step on the staged tensors and reads the output back (one D2H copy).

    As a server overlaps the transfers of one batch with the compute of another, the
    timed loop cycles through R independent batches (their own pages, state and staging
    buffers) on three streams: H2D of step i, compute of step i, D2H of step i, each
    ordered after what it depends on by events.  R is chosen so that the other batches'
    steps touch more than twice the L2 between two uses of one batch (inputs larger than
    L2, no flush inside the timed region).  Whole-job throughput: all ranks' tokens over
    the slowest rank's time."""
    step_bytes = runner.decode_bytes_per_step(w)
    R = max(4, math.ceil(2 * L2_BYTES / max(step_bytes, 1)) + 1)
    batches = []
    for _ in range(R):
        ps = runner.PagedDecodeState(w, st.x)
        parts = [("pos", ps.pos)] + [(k, v) for k, v in ps.new.items()] + [("q", st.x["q"])]
        if "q_I" in st.x:
            parts += [("q_I", st.x["q_I"]), ("w", st.x["w"])]
        # one staging layout shared by host and device: each part 256-byte aligned
        offs, off = {}, 0
        for n, v in parts:
            offs[n] = off
            off += (v.numel() * v.element_size() + 255) // 256 * 256
        hstage = torch.empty(off, dtype=torch.uint8).pin_memory()
        dstage = torch.empty(off, dtype=torch.uint8, device="cuda")

        def view(buf, n, v, offs=offs):
            nb = v.numel() * v.element_size()
            return buf[offs[n]:offs[n] + nb].view(v.dtype).view(v.shape)

        for n, v in parts:
            view(hstage, n, v).copy_(v.contiguous().cpu())
        dv = {n: view(dstage, n, v) for n, v in parts}
        ps.pos = dv["pos"]
        new = {k: dv[k] for k in ps.new}
        hout = torch.empty(ps.out.shape, dtype=ps.out.dtype).pin_memory()
        ev = {k: torch.cuda.Event() for k in ("h2d", "done", "d2h")}
        batches.append(dict(ps=ps, dv=dv, new=new, hstage=hstage, dstage=dstage, hout=hout, ev=ev))
    h2d = batches[0]["hstage"].numel()          # the staging buffer crosses whole (256-byte parts)
    d2h = batches[0]["hout"].numel() * batches[0]["hout"].element_size()
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def step_of(bt, st=None):
        dv = bt["dv"]
        bt["ps"].step(stream if st is None else st, q=dv["q"], q_I=dv.get("q_I"), w_=dv.get("w"),
                      new=bt["new"])

    # each batch's step (its kernel launches) captured once as a CUDA graph, so the host
    # issues one graph launch per step instead of the step's launches
    graphs = None
    try:
        cap = torch.cuda.Stream()
        gs = []
        for bt in batches:
            bt["dstage"].copy_(bt["hstage"])     # the step's inputs (positions included)
        torch.cuda.synchronize()
        for bt in batches:
            step_of(bt, cap)                     # warm the launch path on the capture stream
        torch.cuda.synchronize()
        for bt in batches:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
                step_of(bt, cap)
            gs.append(g)
        torch.cuda.synchronize()
        graphs = gs
    except Exception:   # a launch path that cannot be captured: plain launches
        torch.cuda.synchronize()
        graphs = None

    def one(i):
        bt = batches[i % R]
        e = bt["ev"]
        s_h2d.wait_event(e["done"])              # the batch's previous step has read its staging
        with torch.cuda.stream(s_h2d):
            bt["dstage"].copy_(bt["hstage"], non_blocking=True)
        e["h2d"].record(s_h2d)
        stream.wait_event(e["h2d"])
        stream.wait_event(e["d2h"])              # its previous output has been read back
        if graphs is not None:
            with torch.cuda.stream(stream):
                graphs[i % R].replay()
        else:
            step_of(bt)
        e["done"].record(stream)
        s_d2h.wait_event(e["done"])
        with torch.cuda.stream(s_d2h):
            bt["hout"].copy_(bt["ps"].out, non_blocking=True)
        e["d2h"].record(s_d2h)

    def run(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(stream)
        s_h2d.wait_event(t0)
        for i in range(n):
            one(i)
        stream.wait_stream(s_d2h)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n

    run(2 * R)                                   # warm-up
    dev_times = timed_loop(lambda: step_of(batches[0]), steps, flush, stream)
    barrier(world)
    n = max(steps, 4 * R)
    ms_local = float(np.median([run(n) for _ in range(3)]))
    ms, _, value = aggregate(ms_local, w.b, world)   # whole job, slowest rank
    res = {"value": value, "unit": "tok/s", "h2d_bytes_per_step": int(h2d),
           "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 4),
           "copies_per_step": {"h2d": 1, "d2h": 1},
           "call": "csa_decode_paged (pages of %d entries, state rings)" % L.PAGE_ENTRIES,
           "pipeline": "%d batches in rotation; H2D, step%s and D2H on three streams, "
                       "ordered by events; no L2 flush (the batches' data exceed L2)"
                       % (R, " (one CUDA graph per batch)" if graphs is not None else ""),
           "device_ms_per_step": round(float(np.mean(dev_times)), 4),
           "gpu_launches_per_step": L.csa_decode_paged_launch_count(batches[0]["ps"].p)}
    del batches
    return res


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------

def measure_tc_peaks(peaks):
    """Dense FP8 tensor-core peak of this GPU, measured here: torch._scaled_mm (a plain library
    GEMM) of two 8192 x 8192 E4M3 matrices into bf16, best of 10 after warm-up, 2 N^3 FLOPs.
    Falls back to twice the bf16 peak (the nominal ratio) when the call is not available."""
    n = 8192
    try:
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda")
        f = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)  # noqa: E731
        for _ in range(5):
            f()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        fp8 = 2.0 * n ** 3 / (best * 1e-3) / 1e12
        del a, b
        torch.cuda.empty_cache()
        return {"fp8_tflops": round(fp8, 1), "fp8_src": "measured: torch._scaled_mm e4m3 8192^3, best of 10"}
    except Exception as e:   # noqa: BLE001
        return {"fp8_tflops": 2.0 * peaks["bf16"],
                "fp8_src": "2 x bf16 (nominal ratio): _scaled_mm unavailable (%s)" % type(e).__name__}


def stage_times_prefill(w, st, steps, flush, stream):
    """Mean ms of each stage call of the prefill, each timed alone with events."""
    x = st.x
    E = w.E
    res = {}
    cp = runner.compress_params(w, "main")
    ci = runner.compress_params(w, "index")
    res["compress"] = np.mean(timed_loop(lambda: (
        L.csa_compress(cp, x["C_a"], x["Z_a"], x["B_a"], x["C_b"], x["Z_b"], x["B_b"], w.b, w.n, 0,
                       E, E, st.kv_cache, None, stream),
        L.csa_compress(ci, x["CI_a"], x["ZI_a"], x["BI_a"], x["CI_b"], x["ZI_b"], x["BI_b"], w.b,
                       w.n, 0, E, E, st.kI_cache, st.kI_scales, stream)), steps, flush, stream,
        warm=2))
    rows = w.b * w.n
    codes = torch.empty((rows * w.H_I, runner.row_bytes(w.idx_dtype, w.c_I)), dtype=torch.uint8,
                        device="cuda")
    qs = torch.empty((rows * w.H_I,), dtype=torch.float32, device="cuda")
    res["quantize"] = np.mean(timed_loop(lambda: L.csa_quantize(
        L.DTYPE[w.dtype], L.DTYPE[w.idx_dtype], x["q_I"], rows * w.H_I, w.c_I, codes, qs, stream),
        steps, flush, stream, warm=2))
    qpos = torch.arange(w.n, dtype=torch.int32, device="cuda").repeat(w.b, 1).contiguous()
    scores = torch.empty((w.b, w.n, E), dtype=torch.bfloat16, device="cuda")
    ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[w.idx_dtype],
                       score_dtype=L.CSA_BF16)
    res["index_scores"] = np.mean(timed_loop(lambda: L.csa_index_scores(
        ip, codes, qs, x["w"], st.kI_cache, st.kI_scales, qpos, w.b, w.n, E, E, scores, stream),
        steps, flush, stream, warm=2))
    tkb = L.csa_topk_workspace_size(L.CSA_BF16, w.b, w.n, E, w.k)
    tkws = torch.empty((max(tkb, 256),), dtype=torch.uint8, device="cuda")
    res["topk"] = np.mean(timed_loop(lambda: L.csa_topk(
        scores, L.CSA_BF16, qpos, w.m, w.b, w.n, E, w.k, st.idx, st.count, tkws, tkb, stream),
        steps, flush, stream, warm=2))
    del scores
    ap = L.AttnParams(H=w.H, d=w.c, n_w=w.n_w, scale=w.scale, m=w.m, k=w.k, dtype=L.DTYPE[w.dtype])
    wsb = L.csa_sparse_attn_workspace_size(ap, w.b, w.n, E)
    ws = torch.empty((max(wsb, 256),), dtype=torch.uint8, device="cuda")
    res["sparse_attn"] = np.mean(timed_loop(lambda: L.csa_sparse_attn(
        ap, x["q"], st.kv_cache, E, st.idx, st.count, x["C_a"], w.n, qpos, x["sink"], w.b, w.n,
        st.out, None, ws, wsb, stream), steps, flush, stream, warm=2))
    return {k: float(v) for k, v in res.items()}


def bench_prefill(w, args, world, rank, peaks, min_span_s):
    stream = torch.cuda.current_stream()
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PrefillState(w, inp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for _ in range(args.warmup):
        st.run(stream)
    torch.cuda.synchronize()
    reps, t0, t1 = timed_region(lambda: st.run(stream), args.steps, flush, stream, world,
                                min_span_s)
    ck = clocks.stop(t0, t1)
    ck["repeats"] = len(reps)
    ms, tokens, value = aggregate(float(np.median(reps)), w.b * w.n, world)
    f_idx, f_attn = runner.prefill_flops(w)
    p_fp8, p_bf16 = peaks["fp8"], peaks["bf16"]
    # dtype-weighted: FP8 FLOPs count at the bf16 / FP8 peak ratio, so that achieved / peak is
    # the ideal time at each dtype's peak over the measured time
    t_ideal = f_idx / (p_fp8 * 1e12) + f_attn / (p_bf16 * 1e12)
    weighted = (f_idx * p_bf16 / p_fp8 + f_attn) / (ms * 1e-3) / 1e12
    stage = stage_times_prefill(w, st, max(2, min(args.steps, 5)), flush, stream)
    eb = 2 if w.dtype == "bf16" else 4
    E = w.E
    cbytes = w.b * (4 * w.n * (w.c + w.c_I) * eb + E * w.c * eb + E * (w.c_I + 4))
    qbytes = w.b * w.n * w.H_I * (w.c_I * eb + w.c_I + 4)
    tbytes = w.b * w.n * (E * 2 + (w.k + 1) * 4)
    kernels = {
        "compress": kernel_record(stage["compress"] * 1e3, cbytes, peaks["hbm"]),
        "quantize": kernel_record(stage["quantize"] * 1e3, qbytes, peaks["hbm"]),
        "index_scores": kernel_record(stage["index_scores"] * 1e3, f_idx, p_fp8, "TFLOP/s",
                                      "tensor"),
        "topk": kernel_record(stage["topk"] * 1e3, tbytes, peaks["hbm"]),
        "sparse_attn": kernel_record(stage["sparse_attn"] * 1e3, f_attn, p_bf16, "TFLOP/s",
                                     "tensor"),
    }
    del st, inp, flush
    torch.cuda.empty_cache()
    return dict(value=value, ms=ms, tokens_per_step=tokens, clocks=ck, stage=stage,
                roofline={"bound": "tensor", "achieved": round(weighted, 1), "peak": p_bf16,
                          "unit": "TFLOP/s", "frac": round(t_ideal / (ms * 1e-3), 4),
                          "traffic": None,
                          "kernel": "index_scores + sparse_attn (dtype-weighted, whole prefill)",
                          "achieved_raw_tflops": round((f_idx + f_attn) / (ms * 1e-3) / 1e12, 1),
                          "flops_index_fp8": f_idx, "flops_attn_bf16": f_attn,
                          "peak_fp8": p_fp8, "frac_vs_sustained_bf16":
                          round((f_idx / (p_fp8 * peaks["bf16_sus"] / p_bf16) +
                                 f_attn / peaks["bf16_sus"]) / 1e12 / (ms * 1e-3), 4)},
                kernels=kernels, e2e=None,
                launches=runner.prefill_launches(w) * args.steps * len(reps), repeats=len(reps))


# ---------------------------------------------------------------------------
# reference arm / cpu baseline: the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------

class HostRows:
    """Row access to one sequence of a host tensor, converted to float64 only for the rows
    indexed (so the oracle can walk 1M-token inputs without a float64 copy of them)."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, key):
        if isinstance(key, np.ndarray):
            key = torch.from_numpy(np.asarray(key, dtype=np.int64))
        return self.t[key].double().numpy()

    def __len__(self):
        return self.shape[0]


def oracle_decode_rate(w, budget_s=20.0):
    """tok/s of the oracle's decode step on this host's cores, on sampled sequences.

    The caches (the state a step starts from) are built before timing; the
    timed step compresses the new entry, quantises q_I, scores every entry,
    selects top-k and attends over the selection and the window.
    """
    from oracle import csa, pipeline

    inp = synth.make_inputs(workloads.shrink(w, b=1), device="cpu")
    g = {k: (HostRows(v[0]) if v.dim() >= 3 else v.double().numpy()) for k, v in inp.items()}
    t = w.n - 1
    E = w.E
    main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=g["B_a"], C_b=g.get("C_b"), Z_b=g.get("Z_b"),
                B_b=g.get("B_b"))
    hca = w.kind == "hca_decode"
    q = g["q"][0]
    if not hca:
        index = dict(C_a=g["CI_a"], Z_a=g["ZI_a"], B_a=g["BI_a"], C_b=g["CI_b"], Z_b=g["ZI_b"],
                     B_b=g["BI_b"])
        qI, wI = g["q_I"][0], g["w"][0]
        kI = csa.compress_range(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                index["Z_b"], index["B_b"], w.m, True, 0, E - 1, w.d_rope_I,
                                w.theta, w.eps, chunk_rows=1 << 16)
        kI_deq, _ = pipeline.quantize_rows(kI, w.idx_dtype)
        # the latent cache is state: only the rows a step can gather are filled in
        nk = csa.compress_entries(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                  index["Z_b"], index["B_b"], w.m, True, [E - 1], w.d_rope_I,
                                  w.theta, w.eps)
        qd, _ = pipeline.quantize_rows(qI[None], w.idx_dtype)
        kd = np.concatenate([kI_deq, pipeline.quantize_rows(nk, w.idx_dtype)[0]])
        sc = csa.index_scores(qd, wI[None], kd, np.array([t]), w.m, "bf16")
        sel0 = csa.topk(sc, np.array([t]), w.m, w.k)[0][0]
        sel0 = sel0[(sel0 >= 0) & (sel0 < E - 1)]
        kv_cache = np.zeros((E - 1, w.c))
        kv_cache[sel0] = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                              main["Z_b"], main["B_b"], w.m, True, sel0, w.d_rope,
                                              w.theta, w.eps)
    else:
        kv_cache = csa.compress_range(main["C_a"], main["Z_a"], main["B_a"], None, None, None,
                                      w.m, False, 0, E - 1, w.d_rope, w.theta, w.eps,
                                      chunk_rows=1 << 16)
    win = g["C_a"][csa.window_rows(t, w.n_w)]

    def step():
        new = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"], main["Z_b"],
                                   main["B_b"], w.m, not hca, [E - 1], w.d_rope, w.theta, w.eps)
        kv = np.concatenate([kv_cache, pipeline.round_out(new, w.dtype)])
        if hca:
            rows = np.concatenate([kv, win])
        else:
            nk = csa.compress_entries(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                      index["Z_b"], index["B_b"], w.m, True, [E - 1], w.d_rope_I,
                                      w.theta, w.eps)
            nkd, _ = pipeline.quantize_rows(nk, w.idx_dtype)
            kd = np.concatenate([kI_deq, nkd])
            qd, _ = pipeline.quantize_rows(qI[None], w.idx_dtype)
            sc = csa.index_scores(qd, wI[None], kd, np.array([t]), w.m, "bf16")
            idx, cnt = csa.topk(sc, np.array([t]), w.m, w.k)
            sel = idx[0, :cnt[0]]
            rows = np.concatenate([kv[sel], win])
        return csa.attend(q, rows, g["sink"], w.scale)

    step()
    n, t0, c0 = 0, time.perf_counter(), time.process_time()
    while True:
        step()
        n += 1
        el = time.perf_counter() - t0
        if el > budget_s or n >= w.b:
            break
    par = (time.process_time() - c0) / el
    return n / el, "%d decode step(s) of one sequence (context %d), caches prebuilt" % (n, w.n), par


def oracle_prefill_rate(w, budget_s=20.0):
    from oracle import pipeline
    inp = synth.make_inputs(w, device="cpu")
    g = {k: (v[0] if v.dim() >= 3 else v).double().numpy() for k, v in inp.items()}
    main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=g["B_a"], C_b=g["C_b"], Z_b=g["Z_b"], B_b=g["B_b"])
    index = dict(C_a=g["CI_a"], Z_a=g["ZI_a"], B_a=g["BI_a"], C_b=g["CI_b"], Z_b=g["ZI_b"],
                 B_b=g["BI_b"])
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(w.n, size=min(w.n, 64), replace=False))
    t0, c0 = time.perf_counter(), time.process_time()
    pipeline.csa_prefill(main, index, g["q"], g["q_I"], g["w"], g["sink"], m=w.m, d_rope=w.d_rope,
                         theta=w.theta, eps=w.eps, k=w.k, n_w=w.n_w, scale=w.scale,
                         kv_dtype=w.dtype, idx_dtype=w.idx_dtype, score_dtype=w.score_dtype,
                         query_rows=rows)
    el = time.perf_counter() - t0
    par = (time.process_time() - c0) / el
    return len(rows) / el, "%d of %d query rows (whole compressor included)" % (len(rows), w.n), par


def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(w, budget_s=20.0):
    """The oracle timed on this host.  `cores` is the number of threads it kept busy on
    average over the timed run (process CPU time / wall time, at least 1): numpy spreads
    its large contractions over its BLAS threads and runs element-wise work on one."""
    if w.kind == "csa_prefill":
        v, sample, par = oracle_prefill_rate(w, budget_s)
    else:
        v, sample, par = oracle_decode_rate(w, budget_s)
    sample += "; process CPU time / wall time %.1f on a host of %d threads" % (par, host_threads())
    return {"value": round(v, 3), "unit": "tok/s", "cores": max(1, int(round(par))),
            "kind": "oracle", "sample": sample}


# ---------------------------------------------------------------------------

SUB_WORKLOADS = (workloads.CSA_DECODE_1M, workloads.HCA_DECODE_1M, workloads.CSA_PREFILL_32K)

# Grouped output projection (an output epilogue of the attention): 64 heads x 512 in 8
# groups, each projected to 1024 outputs, for the 64K decode batch and the 32K prefill.
OUT_PROJ = dict(H=64, d=512, g=8, d_g=1024)


def bench_out_proj(args, peaks, world):
    """Event-timed csa_out_proj at the decode batch (16 tokens: the 64 MB of bf16 weights
    bound it, HBM roofline) and at the prefill length (32768 tokens: tensor roofline)."""
    H, d, g, d_g = OUT_PROJ["H"], OUT_PROJ["d"], OUT_PROJ["g"], OUT_PROJ["d_g"]
    K = (H // g) * d
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    W = synth.draw("W_o", (g, d_g, K), 7, "cuda", "bf16", spread=1.0 / math.sqrt(K))
    res = {}
    for label, T in (("decode_16_tokens", workloads.CSA_DECODE_64K.b),
                     ("prefill_32768_tokens", workloads.CSA_PREFILL_32K.n)):
        o = synth.draw("q", (T, H, d), 8, "cuda", "bf16")
        y = torch.empty((T, g * d_g), dtype=torch.bfloat16, device="cuda")
        wsb = L.csa_out_proj_workspace_size(T, H, d, g, d_g)
        ws = torch.empty((max(wsb, 256),), dtype=torch.uint8, device="cuda")
        fn = lambda: L.csa_out_proj(o, W, T, H, d, g, d_g, y, ws, wsb, stream)  # noqa: E731
        us = float(np.mean(timed_loop(fn, max(3, min(args.steps, 10)), flush, stream, warm=3))) * 1e3
        if T <= 64:
            nbytes = W.numel() * 2 + o.numel() * 2 + y.numel() * 2
            res[label] = kernel_record(us, nbytes, peaks["hbm"])
        else:
            res[label] = kernel_record(us, 2.0 * T * K * d_g * g, peaks["bf16"], "TFLOP/s", "tensor")
        res[label]["launches"] = L.lib().csa_out_proj_workspace_size(T, H, d, g, d_g) and 2 or 1
        del o, y, ws
    del W, flush
    torch.cuda.empty_cache()
    res["config"] = dict(OUT_PROJ)
    return res


def bench_csa2(args, peaks, world, w):
    """CSA2 decode modes at a CSA decode workload, each a whole csa_decode call timed with
    events (L2 flushed before each): Full (indexer over every entry, top-k), Reuse (an
    earlier layer's selection: no indexer, no top-k) and Reindex (the indexer and top-k over
    a candidate pool of P = 2k entries per sequence, the earlier layer's top-P)."""
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    inp = synth.make_inputs(w, device="cuda")
    st = runner.DecodeState(w, inp)
    st.build_caches(stream)
    st.step(stream)                                   # layer 1: its selection and caches
    torch.cuda.synchronize()
    idx1, cnt1 = st.idx.clone(), st.count.clone()
    E, P = w.E, 2 * w.k
    # layer 1's top-P of its own scores: the Reindex pool
    ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[w.idx_dtype],
                       score_dtype=L.CSA_BF16)
    codes = torch.empty((w.b * w.H_I, runner.row_bytes(w.idx_dtype, w.c_I)), dtype=torch.uint8,
                        device="cuda")
    qs = (torch.empty((w.b * w.H_I,), dtype=torch.float32, device="cuda") if w.idx_dtype == "fp8"
          else torch.empty((w.b * w.H_I, w.c_I // 16), dtype=torch.uint8, device="cuda"))
    L.csa_quantize(L.DTYPE[w.dtype], L.DTYPE[w.idx_dtype], inp["q_I"], w.b * w.H_I, w.c_I, codes,
                   qs, stream)
    qpos = torch.full((w.b, 1), w.n - 1, dtype=torch.int32, device="cuda")
    sc1 = torch.empty((w.b, 1, E), dtype=torch.bfloat16, device="cuda")
    L.csa_index_scores(ip, codes, qs, inp["w"], st.kI_cache, st.kI_scales, qpos, w.b, 1, st.E_cap,
                       E, sc1, stream)
    pool = torch.empty((w.b, 1, P), dtype=torch.int32, device="cuda")
    pcnt = torch.empty((w.b, 1), dtype=torch.int32, device="cuda")
    tkb = L.csa_topk_workspace_size(L.CSA_BF16, w.b, 1, E, P)
    tkws = torch.empty((max(tkb, 256),), dtype=torch.uint8, device="cuda")
    L.csa_topk(sc1, L.CSA_BF16, qpos, w.m, w.b, 1, E, P, pool, pcnt, tkws, tkb, stream)
    res = {}
    for label, mode in (("full", L.CSA_MODE_FULL), ("reuse", L.CSA_MODE_REUSE),
                        ("reindex", L.CSA_MODE_REINDEX)):
        p = runner.decode_params(w, st.E_cap)
        p.mode, p.P = mode, (P if mode == L.CSA_MODE_REINDEX else 0)
        t = st.tensors()
        t["out"] = torch.empty_like(st.out)
        t["idx_out"] = torch.empty((w.b, w.k), dtype=torch.int32, device="cuda")
        t["count_out"] = torch.empty((w.b,), dtype=torch.int32, device="cuda")
        if mode == L.CSA_MODE_REUSE:
            t["idx_in"], t["count_in"] = idx1, cnt1
        if mode == L.CSA_MODE_REINDEX:
            t["pool"], t["pool_count"] = pool.reshape(w.b, P), pcnt.reshape(w.b)
        wsb = L.csa_decode_workspace_size(p)
        ws = torch.empty((max(wsb, 256),), dtype=torch.uint8, device="cuda")
        fn = lambda: L.csa_decode(p, t, ws, wsb, stream)  # noqa: E731
        us = float(np.median(timed_loop(fn, max(5, min(args.steps, 20)), flush, stream, warm=3))) * 1e3
        res[label] = {"us_per_step": round(us, 2), "tok_s": round(w.b / (us * 1e-6), 1),
                      "launches": L.csa_decode_launch_count(p)}
        del ws
    if L.csa_device_error():
        raise RuntimeError("device error word set during the CSA2 measurement")
    del st, inp, flush
    torch.cuda.empty_cache()
    res["config"] = {"workload": w.name, "batch": w.b, "context": w.n, "top_k": w.k, "pool": P}
    return res


def bench_cp(args, peaks, world, G=8):
    """One rank's share of a context-parallel 1M CSA decode over G ranks (1M workload, the
    entries of every sequence split into G shards), timed on this GPU phase by phase with
    events (L2 flushed before each): the local phase (compress the new entry on the rank that
    holds it, quantise, score the shard, its top-k, candidates), the merge of the gathered
    candidates and the packing of the rows this rank holds, and the attention over the k
    gathered rows and the window.  The two collectives between them move the bytes given in
    `exchange_bytes` (all-gather of the candidates, all-reduce of the packed rows); one GPU
    does not measure them."""
    from long_context_sparse_05_b200 import cp as cpmod
    w = workloads.CSA_DECODE_1M
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    inp = synth.make_inputs(w, device="cuda")
    full = runner.DecodeState(w, inp)
    full.build_caches(stream)
    torch.cuda.synchronize()
    shard = cpmod.CPShard(w, inp, G - 1, G, full)     # the rank that completes the new entry
    del full
    torch.cuda.empty_cache()
    shard.phase_local(stream)
    for r in range(G):                                # every rank's candidates: this rank's
        shard.gath_s[r].copy_(shard.cand_s)
        shard.gath_i[r].copy_(shard.cand_i)
    steps = max(5, min(args.steps, 20))
    res = {}
    for label, fn in (("local", lambda: shard.phase_local(stream)),
                      ("merge_pack", lambda: shard.phase_merge(stream)),
                      ("attend", lambda: shard.phase_attend(stream))):
        res[label + "_us"] = round(float(np.median(timed_loop(fn, steps, flush, stream, warm=3))) * 1e3, 2)
    if L.csa_device_error():
        raise RuntimeError("device error word set during the context-parallel measurement")
    res["rank_us_without_collectives"] = round(res["local_us"] + res["merge_pack_us"] + res["attend_us"], 2)
    res["exchange_bytes"] = {"all_gather_candidates": G * w.b * w.k * (2 + 4),
                             "all_reduce_rows": w.b * w.k * w.c * 2}
    res["config"] = {"workload": w.name, "ranks": G, "rank": G - 1, "shard_entries": shard.n_local,
                     "batch": w.b, "context": w.n, "top_k": w.k}
    del shard, inp, flush
    torch.cuda.empty_cache()
    return res


def run_workload(w, args, world, rank, peaks, min_span_s, cpu_budget_s):
    """One workload's record: throughput, rooflines, per-kernel fractions, clocks, e2e and (rank
    0 of a single-GPU run) the oracle's rate on this host."""
    if w.kind == "csa_prefill":
        r = bench_prefill(w, args, world, rank, peaks, min_span_s)
    else:
        r = bench_decode(w, args, world, rank, peaks, min_span_s)
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, cpu_budget_s)
    rec = {"value": round(r["value"], 2), "unit": "tok/s", "ms_per_step": round(r["ms"], 5),
           "steps": args.steps, "repeats": r["repeats"],
           "dtype": w.dtype + ("+" + w.idx_dtype if w.c_I else ""),
           "config": {"workload": w.name, "batch_per_gpu": w.b, "context": w.n, "m": w.m,
                      "top_k": w.k, "window": w.n_w, "heads": w.H, "latent": w.c,
                      "index_heads": w.H_I, "index_dim": w.c_I, "parallelism":
                      "replicas%d" % world, "l2": "flushed (256 MiB write) before each step"},
           "roofline": r["roofline"], "kernels": r["kernels"], "cpu_baseline": cb,
           "e2e": r["e2e"], "gpu_launches": r["launches"], "clocks": r["clocks"],
           "stage_us": {k: round(v * 1e3, 2) for k, v in r["stage"].items()}}
    if "step_roofline" in r:
        rec["step_roofline"] = r["step_roofline"]
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=sorted(workloads.ALL),
                    help="run only this workload (default: the 64K CSA decode headline plus "
                         "the 1M CSA / HCA decode and 32K prefill sub-records)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-span", type=float, default=1.0,
                    help="seconds the repeated timed region of the headline spans at least")
    ap.add_argument("--context", type=int, default=0,
                    help="override the context length (profiling of a smaller case, not a bench line)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = workloads.ALL[args.workload or workloads.CSA_DECODE_64K.name]
    if args.context:
        w = workloads.shrink(w, n=args.context)
    if args.batch:
        w = workloads.shrink(w, b=args.batch)
    peaks = load_peaks()

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        cb = cpu_baseline(w)
        line = {"metric": METRIC, "value": cb["value"], "unit": "tok/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": w.name, "batch": w.b, "context": w.n},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    world, rank, local = dist_setup(args.gpus)
    L.lib()
    peaks.update(measure_tc_peaks(peaks))
    peaks["fp8"] = peaks["fp8_tflops"]
    head = run_workload(w, args, world, rank, peaks, args.min_span, 20.0)
    subs = {}
    if args.workload is None and not args.context and not args.batch:
        for w2 in SUB_WORKLOADS:
            subs[w2.name] = run_workload(w2, args, world, rank, peaks, 0.5, 10.0)
        subs["grouped_out_proj"] = bench_out_proj(args, peaks, world)
        subs["csa2_modes_64k"] = bench_csa2(args, peaks, world, workloads.CSA_DECODE_64K)
        subs["csa2_modes_1m"] = bench_csa2(args, peaks, world, workloads.CSA_DECODE_1M)
        subs["context_parallel_1m_rank"] = bench_cp(args, peaks, world)
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": "tok/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": head["dtype"], "data": "synthetic"}
        line.update({k: v for k, v in head.items() if k not in line})
        line["peaks"] = {"src": peaks["src"], "hbm_gbs": peaks["hbm"], "bf16_tflops": peaks["bf16"],
                         "bf16_tflops_sustained": peaks["bf16_sus"],
                         "fp8_tflops": peaks["fp8"], "fp8_src": peaks["fp8_src"]}
        if subs:
            line["sub"] = subs
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
