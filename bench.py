"""Benchmark of the CSA / HCA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload: CSA decode at 64K context (16 sequences, FP8 indexer,
top-k 512, window 128, 64 heads x 512).  A step is one fused decode step for
the whole batch (compress the entry the new token completes, quantise the
index query, score every entry, select top-k, attend over selection + window)
with inputs resident in HBM.  L2 is flushed (a 256 MiB write) before every
timed step, outside the step's CUDA events.  Multi-GPU runs are independent
replicas (the path has no exchange step): value = all ranks' tokens / max
over ranks of the device time.

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
        for a, b in evs:
            flush_buf.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        if nvtx:
            torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

# DRAM bytes (read + write) per processed key entry of the dominant kernel, from the ncu
# captures under profiles/ (ncu_full_csa_decode_64k_fp8_b4.md: the FP8 indexer at batch 4,
# 16384 entries per sequence; ncu_full_index_scores_fp4_ctx256k_b2.md: the NVFP4 indexer at
# 256K context, batch 2, 65536 entries per sequence). The traffic is linear in the entries, so
# one launch's figure is this times b * E of the launch timed. A kernel changed after its
# capture has no entry here (traffic is then reported as null).
PROFILED_TRAFFIC_PER_ENTRY = {
    ("index_scores", "fp8"): 8717056 / (4 * 16384),
    ("index_scores", "nvfp4"): 9491712 / (2 * 65536),
}


def profiled_traffic(w, kernel):
    per = PROFILED_TRAFFIC_PER_ENTRY.get((kernel, w.idx_dtype))
    return None if per is None else round(per * w.b * w.E)


def bench_decode(w, args, world, rank, peaks):
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

    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    times = timed_loop(step, args.steps, flush, stream, nvtx="timed_steps")
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    ck = clocks.stop(t0, t1)
    ms, tokens_per_step, value = aggregate(float(np.mean(times)), w.b, world)

    # dominant kernel: the indexer over all E entries (same call the step makes)
    stage = stage_times_decode(w, st, args.steps, flush, stream)
    idx_bytes = w.b * w.E * {"fp8": w.c_I + 4, "nvfp4": w.c_I // 2 + w.c_I // 16}.get(
        w.idx_dtype, w.c * 2)
    dom = "index_scores" if w.kind != "hca_decode" else "sparse_attn"
    if w.kind == "hca_decode":
        dom_bytes = w.b * (w.E + w.n_w) * w.c * 2 + 2 * w.b * w.H * w.c * 2
    else:
        dom_bytes = idx_bytes + w.b * w.H_I * (w.c_I + 4 + 4)
    dom_ms = stage[dom]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    step_bytes = runner.decode_bytes_per_step(w)

    e2e = e2e_decode(w, st, args.steps, flush, stream, world)
    return dict(value=value, ms=ms, tokens_per_step=tokens_per_step, clocks=ck, stage=stage,
                roofline={"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"],
                          "unit": "GB/s", "frac": round(achieved / peaks["hbm"], 4),
                          "traffic": profiled_traffic(w, dom), "kernel": dom,
                          "algorithmic_bytes_per_launch": dom_bytes},
                step_roofline={"algorithmic_bytes": step_bytes,
                               "achieved_gbs": round(step_bytes / (ms * 1e-3) / 1e9, 1),
                               "frac": round(step_bytes / (ms * 1e-3) / 1e9 / peaks["hbm"], 4)},
                e2e=e2e, launches=runner.decode_launches_per_step(w) * args.steps)


def stage_times_decode(w, st, steps, flush, stream):
    """Mean µs of each stage call of the decode step, each timed alone with events."""
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


def e2e_decode(w, st, steps, flush, stream, world=1):
    """Same step through the public API with host inputs: every step copies its new
    inputs (q, q_I, w and the m raw rows of the completing block of every C / Z
    tensor) from one pinned host buffer to one device staging buffer (a single H2D
    copy), places the raw rows into the sequence tensors with device-to-device
    copies, runs the decode call on the staged q / q_I / w, and reads the output back
    (one D2H copy).  Whole-job throughput: all ranks' tokens over the slowest rank's
    time."""
    x = st.x
    t = w.n - 1
    r0 = t - (w.m - 1)
    names = ["C_a", "Z_a", "C_b", "Z_b", "CI_a", "ZI_a", "CI_b", "ZI_b"]
    names = [n for n in names if n in x]
    parts = [("q", x["q"])]
    if "q_I" in x:
        parts += [("q_I", x["q_I"]), ("w", x["w"])]
    parts += [(n, x[n][:, r0:t + 1]) for n in names]
    # one staging layout shared by host and device: each part 256-byte aligned
    offs, off = {}, 0
    for n, v in parts:
        offs[n] = off
        off += (v.numel() * v.element_size() + 255) // 256 * 256
    hstage = torch.empty(off, dtype=torch.uint8).pin_memory()
    dstage = torch.empty(off, dtype=torch.uint8, device="cuda")

    def view(buf, n, v):
        nb = v.numel() * v.element_size()
        return buf[offs[n]:offs[n] + nb].view(v.dtype).view(v.shape)

    for n, v in parts:
        view(hstage, n, v).copy_(v.contiguous().cpu())
    dviews = {n: view(dstage, n, v) for n, v in parts}
    hout = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for _, v in parts)
    d2h = hout.numel() * hout.element_size()

    def one():
        dstage.copy_(hstage, non_blocking=True)
        for n in names:
            x[n][:, r0:t + 1].copy_(dviews[n])
        st.step(stream, q=dviews["q"], q_I=dviews.get("q_I"), w_=dviews.get("w"))
        hout.copy_(st.out, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    barrier(world)
    times = timed_loop(one, steps, flush, stream)
    ms, _, value = aggregate(float(np.mean(times)), w.b, world)   # whole job, slowest rank
    return {"value": value, "unit": "tok/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 4),
            "copies_per_step": {"h2d": 1, "d2d": len(names), "d2h": 1}}


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------

def bench_prefill(w, args, world, rank, peaks):
    stream = torch.cuda.current_stream()
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PrefillState(w, inp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for _ in range(args.warmup):
        st.run(stream)
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.time()
    times = timed_loop(lambda: st.run(stream), args.steps, flush, stream, nvtx="timed_steps")
    t1 = time.time()
    barrier(world)
    ck = clocks.stop(t0, t1)
    ms, tokens, value = aggregate(float(np.mean(times)), w.b * w.n, world)
    f_idx, f_attn = runner.prefill_flops(w)
    p_fp8 = 2 * peaks["bf16"]
    t_ideal = f_idx / (p_fp8 * 1e12) + f_attn / (peaks["bf16"] * 1e12)
    frac = t_ideal / (ms * 1e-3)
    return dict(value=value, ms=ms, tokens_per_step=tokens, clocks=ck, stage={},
                roofline={"bound": "tensor", "achieved": round(
                    (f_idx + f_attn) / (ms * 1e-3) / 1e12, 2), "peak": peaks["bf16"],
                    "unit": "TFLOP/s", "frac": round(frac, 4), "traffic": None,
                    "kernel": "whole prefill (dtype-weighted)",
                    "flops_index_fp8": f_idx, "flops_attn_bf16": f_attn},
                e2e=None, launches=runner.prefill_launches(w) * args.steps)


# ---------------------------------------------------------------------------
# reference arm / cpu baseline: the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------

def oracle_decode_rate(w, budget_s=20.0):
    """tok/s of the oracle's decode step on this host's cores, on sampled sequences.

    The caches (the state a step starts from) are built before timing; the
    timed step compresses the new entry, quantises q_I, scores every entry,
    selects top-k and attends over the selection and the window.
    """
    from oracle import codecs, csa, pipeline

    inp = synth.make_inputs(workloads.shrink(w, b=1), device="cpu")
    g = {k: (v[0] if v.dim() >= 3 else v).double().numpy() for k, v in inp.items()}
    t = w.n - 1
    E = w.E
    main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=g["B_a"], C_b=g.get("C_b"), Z_b=g.get("Z_b"),
                B_b=g.get("B_b"))
    hca = w.kind == "hca_decode"
    if not hca:
        index = dict(C_a=g["CI_a"], Z_a=g["ZI_a"], B_a=g["BI_a"], C_b=g["CI_b"], Z_b=g["ZI_b"],
                     B_b=g["BI_b"])
        kI = csa.compress_range(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                index["Z_b"], index["B_b"], w.m, True, 0, E - 1, w.d_rope_I,
                                w.theta, w.eps, chunk_rows=1 << 14)
        kI_deq, _ = pipeline.quantize_rows(kI, w.idx_dtype)
        # the latent cache is state: only the rows a step can gather are filled in
        nk = csa.compress_entries(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                  index["Z_b"], index["B_b"], w.m, True, [E - 1], w.d_rope_I,
                                  w.theta, w.eps)
        qd, _ = pipeline.quantize_rows(g["q_I"][0][None], w.idx_dtype)
        kd = np.concatenate([kI_deq, pipeline.quantize_rows(nk, w.idx_dtype)[0]])
        sc = csa.index_scores(qd, g["w"][0][None], kd, np.array([t]), w.m, "bf16")
        sel0 = csa.topk(sc, np.array([t]), w.m, w.k)[0][0]
        sel0 = sel0[(sel0 >= 0) & (sel0 < E - 1)]
        kv_cache = np.zeros((E - 1, w.c))
        kv_cache[sel0] = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                              main["Z_b"], main["B_b"], w.m, True, sel0, w.d_rope,
                                              w.theta, w.eps)
    else:
        kv_cache = csa.compress_range(main["C_a"], main["Z_a"], main["B_a"], None, None, None,
                                      w.m, False, 0, E - 1, w.d_rope, w.theta, w.eps,
                                      chunk_rows=1 << 14)

    def step():
        new = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"], main["Z_b"],
                                   main["B_b"], w.m, not hca, [E - 1], w.d_rope, w.theta, w.eps)
        kv = np.concatenate([kv_cache, pipeline.round_out(new, w.dtype)])
        if hca:
            rows = np.concatenate([kv, g["C_a"][csa.window_rows(t, w.n_w)]])
        else:
            nk = csa.compress_entries(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                      index["Z_b"], index["B_b"], w.m, True, [E - 1], w.d_rope_I,
                                      w.theta, w.eps)
            nkd, _ = pipeline.quantize_rows(nk, w.idx_dtype)
            kd = np.concatenate([kI_deq, nkd])
            qd, _ = pipeline.quantize_rows(g["q_I"][0][None], w.idx_dtype)
            sc = csa.index_scores(qd, g["w"][0][None], kd, np.array([t]), w.m, "bf16")
            idx, cnt = csa.topk(sc, np.array([t]), w.m, w.k)
            sel = idx[0, :cnt[0]]
            rows = np.concatenate([kv[sel], g["C_a"][csa.window_rows(t, w.n_w)]])
        return csa.attend(g["q"][0], rows, g["sink"], w.scale)

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

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=workloads.CSA_DECODE_64K.name,
                    choices=sorted(workloads.ALL))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--context", type=int, default=0,
                    help="override the context length (profiling of a smaller case, not a bench line)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = workloads.ALL[args.workload]
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
    if w.kind == "csa_prefill":
        r = bench_prefill(w, args, world, rank, peaks)
    else:
        r = bench_decode(w, args, world, rank, peaks)
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w)
    if rank == 0:
        line = {"metric": METRIC, "value": round(r["value"], 2), "unit": "tok/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(r["ms"], 5), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": w.dtype + ("+" + w.idx_dtype if w.c_I else ""),
                "data": "synthetic",
                "config": {"workload": w.name, "batch_per_gpu": w.b, "context": w.n, "m": w.m,
                           "top_k": w.k, "window": w.n_w, "heads": w.H, "latent": w.c,
                           "index_heads": w.H_I, "index_dim": w.c_I, "parallelism":
                           "replicas%d" % world, "l2": "flushed (256 MiB write) before each step"},
                "roofline": r["roofline"], "cpu_baseline": cb, "e2e": r["e2e"],
                "gpu_launches": r["launches"], "clocks": r["clocks"],
                "stage_us": {k: round(v * 1e3, 2) for k, v in r["stage"].items()},
                "peaks": peaks["src"]}
        if "step_roofline" in r:
            line["step_roofline"] = r["step_roofline"]
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
