"""Benchmark: chunk-causal attention at the 720p latent shape on B200.

One step = one chunk of the stream at the 720p shape: two denoising-step
attention calls (1620 queries x 24 heads x 128 over sink + 3-chunk window +
current chunk = 8100 keys) and the clean-KV append of the chunk, through the
C ABI of libcca.so.  The ring is prefilled with chunks 0..3, so every step sees
the steady-state visible set (5 chunks).  Metric: algorithmic attention TFLOP/s
(4 * Lq * Lk * H * D per call) over the whole step time, plus ms per chunk.

Inputs are synthetic (seeded, see ``synth``) and resident in HBM when timing
starts.  Steps cycle through 3 independent replicas of the state (~420 MB in
total, more than the 126 MB L2), so no step finds the previous step's data in L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the workload: the method needs no exchange between GPUs ("replicas only"), so
the only collectives are the barriers and the max-over-ranks of the timing.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk-attn TFLOP/s & ms/chunk at 720p latent shape; % of BF16/FP8 tensor peak"
WORKLOAD = ("720p-shaped chunk: 1620 tokens (30x54 latent grid), 24 heads x 128, sink + 3-chunk window "
            "+ current chunk (8100 keys), 2 denoising-step attention calls + clean-KV append per chunk")
L, H, D, W = 1620, 24, 128, 3
LK = (1 + W + 1) * L
FLOP_PER_CALL = 4.0 * L * LK * H * D
CALLS_PER_STEP = 2


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


# ------------------------------------------------------------------ ranks
def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity with one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, flop_per_rank_step: float, ms_per_step_max: float) -> float:
    """Whole-job TFLOP/s: work of all replicas over the slowest rank's time."""
    return world * flop_per_rank_step / (ms_per_step_max * 1e-3) / 1e12


# ------------------------------------------------------------------ clocks
class NvmlClockSampler:
    """SM clock and throttle reasons sampled through NVML every ``period_s``
    during the timed region (dense enough for a region of a few ms)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        import pynvml
        pynvml.nvmlInit()
        self.nv = pynvml
        self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
        self.period = period_s
        self.rows = []
        self.times = []  # time.perf_counter() of each row
        self.stop_flag = False

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.rows.append((float(mhz), float(mx), int(rs)))
                self.times.append(time.perf_counter())
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        time.sleep(0.02)

    def stop(self, n_skip: int = 0):
        time.sleep(0.01)
        self.stop_flag = True
        self.thread.join(timeout=2)
        rows = self.rows[n_skip:] or self.rows
        if not rows:
            return None
        reasons = sorted({n for _, _, r in rows for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_min_mhz": min(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons, "samples": len(rows),
                "sampler": f"NVML every {self.period * 1e3:.0f} ms"}


def clock_sampler(gpu_index: int):
    try:
        return NvmlClockSampler(gpu_index)
    except Exception:
        return ClockSampler(gpu_index)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self, n_skip: int = 0):
        if not self.proc:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        rows = rows[n_skip:] or rows
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle legs
def oracle_sample(n_q_rows: int, n_heads: int, seed: int = 1):
    """Time the fp64 oracle on a bounded sample of the 720p attention call:
    the first ``n_q_rows`` queries of ``n_heads`` heads over all 8100 keys."""
    import synth
    from oracle import chunk_attention as oca
    g = synth.rng(seed)
    shape_q = (n_q_rows, n_heads, D)
    q = g.standard_normal(shape_q).astype(np.float32)
    ks = [g.standard_normal((L, n_heads, D)).astype(np.float32) for _ in range(W + 2)]
    vs = [g.standard_normal((L, n_heads, D)).astype(np.float32) for _ in range(W + 2)]
    t = W + 1
    t0 = time.perf_counter()
    oca.chunk_attention(q, ks, vs, t, W)
    dt = time.perf_counter() - t0
    return 4.0 * n_q_rows * LK * n_heads * D, dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline():
    """The fp64 oracle on the host cores: the 720p call (the line's value), plus
    the tiny stream and the 486-query mask-cached call, each the median of 3 runs."""
    import synth
    from oracle import chunk_attention as oca
    runs = [oracle_sample(L, H) for _ in range(3)]  # one full 720p attention call each
    flop = runs[0][0]
    dt = statistics.median(r[1] for r in runs)
    # tiny stream: 4 chunks of 16 tokens, H=1, D=64, W=2 (all four chunk calls)
    s0 = synth.tiny()
    t0s = []
    for _ in range(3):
        t0 = time.perf_counter()
        for t in range(4):
            oca.chunk_attention(s0.q[t], s0.k, s0.v, t, s0.window)
        t0s.append(time.perf_counter() - t0)
    flop0 = sum(4.0 * 16 * (16 * len(oca.visible_chunks(t, 2))) * 64 for t in range(4))
    # mask-cached call: 486 active queries of the 720p call
    t4s = [oracle_sample(486, H)[1] for _ in range(3)]
    flop4 = 4.0 * 486 * LK * H * D
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle, one full 720p attention call (1620 queries x 24 heads x 8100 keys), "
                      f"median of 3 runs: {dt:.2f} s",
            "workloads": {
                "720p_call": {"s_median": dt, "s_runs": [r[1] for r in runs], "tflops": flop / dt / 1e12},
                "tiny_stream_4_chunks": {"ms_median": statistics.median(t0s) * 1e3,
                                         "ms_runs": [x * 1e3 for x in t0s],
                                         "gflops": flop0 / statistics.median(t0s) / 1e9},
                "mask_cached_486_queries": {"s_median": statistics.median(t4s), "s_runs": t4s,
                                            "tflops": flop4 / statistics.median(t4s) / 1e12}}}


def run_reference(args, rank, world):
    """Reference arm: the oracle as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    rows, heads = 128, 1  # one 128-query tile of one head per step
    for _ in range(args.warmup):
        oracle_sample(rows, heads)
    tot_flop, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        f, dt = oracle_sample(rows, heads)
        tot_flop += f
        tot_t += dt
    value = tot_flop / tot_t / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": L, "kv_len": LK,
                       "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": "each step: 128 queries x 1 head of the 720p call over 8100 keys, fp64 (small "
                                       "products: below the whole-call BLAS throughput of the main line's "
                                       "cpu_baseline)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ extra workloads (rank-local)
def _timed(fn, reps, stream, warm=3):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    # hold the stream while the host queues every rep, so that host-side call
    # overhead never shows between the events of a short kernel
    torch.cuda._sleep(int(reps * 100e-6 * 2e9))
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def extra_workloads(dev, stream, peak_tf, peak_gbs):
    """FP8 720p attention, the mask-cached chunk, the 225-chunk latency drift and
    the memory-bound kernels' bandwidth.  Each is timed with CUDA events."""
    import torch
    import synth
    import chunk_causal_attention_b200 as cca
    bf = lambda x: synth.as_torch_bf16(x, dev)
    out = {}
    # L2 flush between reps: a read of 256 MB leaves L2 full of clean lines, so the
    # timed kernel pays no write-back of the flush's own data
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    # ---- e4m3 attention at the 720p shape (Student-t inputs)
    s3 = synth.fp8_720p(n_steps=1)
    ring8 = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev)
    for t in range(s3.t):
        ring8.append(bf(s3.ring_k[t]), bf(s3.ring_v[t]))
    qb, kb, vb = bf(s3.q[0]), bf(s3.k_cur[0]), bf(s3.v_cur[0])
    q8, qs, k8, ks, v8, vs = cca.cca_quant_e4m3_qkv(qb, kb, vb)
    o8 = torch.empty((L, H, D), dtype=torch.bfloat16, device=dev)
    ws8 = torch.empty(max(cca.cca_chunk_attn_workspace_size(ring8, L), 16), dtype=torch.uint8, device=dev)

    t8 = _timed(lambda: cca.cca_chunk_attn(ring8, q8, k8, v8, q_scale=qs, kcur_scale=ks, vcur_scale=vs,
                                             out=o8, workspace=ws8), 50, stream)
    us8 = float(np.median(t8)) * 1e3
    tq = []
    for _ in range(20):  # the call's input quantisation (Q, K -> codes, V -> fp16-widened codes), L2 flushed
        flush.sum()
        torch.cuda._sleep(200000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        cca.cca_quant_e4m3_qkv(qb, kb, vb)
        b.record(stream)
        torch.cuda.synchronize()
        tq.append(a.elapsed_time(b) * 1e3)
    usq = float(np.median(tq))
    out["fp8_720p"] = {"attn_us_per_call": us8, "tflops": FLOP_PER_CALL / (us8 * 1e-6) / 1e12,
                       "quant_qkv_us": usq, "call_incl_quant_us": us8 + usq,
                       "frac_of_fp8_peak": FLOP_PER_CALL / (us8 * 1e-6) / 1e12 / (2 * peak_tf),
                       "note": "QK^T on e4m3 tensor cores; PV in fp16 (P kept 16-bit) over V as fp16-widened e4m3 values; fp8 peak = 2 x bf16 measured"}

    # ---- mask-cached chunk: mask (dynamic tau) + compaction + active-query attention + scatter
    c1 = synth.chunk_720p(n_steps=1)
    m = synth.mask_chunk()
    ring = cca.KVRing(H, D, L, W, device=dev)
    for t in range(c1.t):
        ring.append(bf(c1.ring_k[t]), bf(c1.ring_v[t]))
    q, kc, vc = bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0])
    src, edit = torch.from_numpy(m.src).to(dev), torch.from_numpy(m.edit).to(dev)
    cache = bf(m.o_cache)
    mask = torch.empty(L, dtype=torch.uint8, device=dev)
    idx = torch.empty(L, dtype=torch.int32, device=dev)
    n_act = torch.empty(1, dtype=torch.int32, device=dev)
    oc = torch.empty((L, H, D), dtype=torch.bfloat16, device=dev)
    wsm = torch.empty(max(cca.cca_chunk_attn_workspace_size(ring, L), 16), dtype=torch.uint8, device=dev)

    def chunk4():
        cca.cca_token_mask_l2(src, edit, prune_quantile=m.prune_quantile, mask=mask)
        cca.cca_compact(mask, idx, n_act)
        cca.cca_chunk_attn(ring, q, kc, vc, q_idx=idx, n_q_dev=n_act, n_q_max=L, out=oc, workspace=wsm)
        cca.cca_scatter(oc, idx, n_act, cache, n_max=L)
    def chunk4_fused():  # the scatter-back fused into the attention epilogue
        cca.cca_token_mask_l2(src, edit, prune_quantile=m.prune_quantile, mask=mask)
        cca.cca_compact(mask, idx, n_act)
        cca.cca_chunk_attn_scatter(ring, q, kc, vc, idx, cache, n_q_dev=n_act, n_q_max=L, workspace=wsm)
    t4 = _timed(chunk4, 50, stream)
    t4f = _timed(chunk4_fused, 50, stream)
    t4a = _timed(lambda: cca.cca_chunk_attn(ring, q, kc, vc, q_idx=idx, n_q_dev=n_act, n_q_max=L, out=oc,
                                            workspace=wsm), 50, stream)
    n_active = int(n_act.item())
    flop4 = 4.0 * n_active * LK * H * D
    out["mask_cached_720p"] = {"n_active": n_active, "ms_per_chunk": float(np.median(t4f)),
                               "ms_per_chunk_separate_scatter": float(np.median(t4)),
                               "attn_us": float(np.median(t4a)) * 1e3,
                               "attn_tflops": flop4 / (float(np.median(t4a)) * 1e-3) / 1e12}

    # ---- long stream: per-chunk latency over 225 chunks (AR(1) K/V made on the device).
    # Three passes (fresh ring each); per-chunk medians over the passes damp
    # clock changes of the shared, power-capped GPU.
    def stream_pass(seed, pace_cycles=0):
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        ring2 = cca.KVRing(H, D, L, W, device=dev)
        xk = torch.randn((L, H, D), generator=gen, device=dev)
        xv = torch.randn((L, H, D), generator=gen, device=dev)
        qq = torch.randn((2, L, H, D), generator=gen, device=dev).to(torch.bfloat16)
        o2 = torch.empty((L, H, D), dtype=torch.bfloat16, device=dev)
        ws2 = torch.empty(max(cca.cca_chunk_attn_workspace_size(ring2, L), 16), dtype=torch.uint8, device=dev)
        lat = []
        for t in range(225):
            kb, vb = xk.to(torch.bfloat16), xv.to(torch.bfloat16)
            if pace_cycles:
                torch.cuda._sleep(pace_cycles)  # an idle gap on the device before the chunk (not timed)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for st in range(CALLS_PER_STEP):
                cca.cca_chunk_attn(ring2, qq[st], kb, vb, out=o2, workspace=ws2)
            ring2.append(kb, vb)
            b.record(stream)
            lat.append((a, b))
            xk = 0.9 * xk + 0.44 * torch.randn((L, H, D), generator=gen, device=dev)
            xv = 0.9 * xv + 0.44 * torch.randn((L, H, D), generator=gen, device=dev)
        torch.cuda.synchronize()
        t_end = time.perf_counter()
        lat_ms = np.array([a.elapsed_time(b) for a, b in lat])
        start_ms = np.array([lat[0][0].elapsed_time(a) for a, _ in lat])  # chunk starts on the GPU's timeline
        span_ms = lat[0][0].elapsed_time(lat[-1][1])
        return lat_ms, start_ms, span_ms, t_end

    def window_mhz(smp, t_end, span_ms, lo_ms, hi_ms):
        """Median SM clock of the samples taken while the GPU ran [lo_ms, hi_ms)
        of a pass (the pass ended at host time t_end, span_ms after it began)."""
        if smp is None:
            return None
        t0 = t_end - span_ms * 1e-3
        sel = [r[0] for r, t in zip(smp.rows, smp.times) if lo_ms <= (t - t0) * 1e3 < hi_ms]
        return float(np.median(sel)) if sel else None
    # A first pass from an idle GPU drifted +6-8 % while the clock settled under the power cap
    # (later passes: within 1 %); it is run as warm-up and not counted.  Each counted pass records
    # the SM clock (NVML) while it runs.
    warm_lat = stream_pass(1)[0]
    pass_clocks = []
    runs = []
    drift_norm = []  # per pass: (time x SM clock) of chunks 200-224 against chunks 5-29
    for k in range(3):
        try:
            smp = NvmlClockSampler(dev.index if dev.index is not None else 0, period_s=0.002)
            smp.start()
        except Exception:
            smp = None
        lat_ms, start_ms, span_ms, t_end = stream_pass(2 + k)
        runs.append(lat_ms)
        pass_clocks.append(smp.stop() if smp else None)
        f_early = window_mhz(smp, t_end, span_ms, start_ms[5], start_ms[30])
        f_late = window_mhz(smp, t_end, span_ms, start_ms[200], start_ms[224] + lat_ms[224])
        if f_early and f_late:
            e, l_ = float(np.median(lat_ms[5:30])) * f_early, float(np.median(lat_ms[200:225])) * f_late
            drift_norm.append({"pct": (l_ - e) / e * 100.0, "sm_mhz_5_29": f_early, "sm_mhz_200_224": f_late})
        else:
            drift_norm.append(None)
    passes = np.stack(runs)
    ms = np.median(passes, axis=0)
    early, late = float(np.median(ms[5:30])), float(np.median(ms[200:225]))
    slope = float(np.polyfit(np.arange(5, 225), ms[5:225], 1)[0])
    drift_each = [float((np.median(p[200:225]) - np.median(p[5:30])) / np.median(p[5:30]) * 100) for p in passes]
    out["long_stream_225"] = {"ms_per_chunk_median_5_29": early, "ms_per_chunk_median_200_224": late,
                              "drift_pct": (late - early) / early * 100.0, "drift_pct_each_pass": drift_each,
                              "ols_slope_ms_per_chunk": slope, "first_chunks_ms": [float(x) for x in ms[:5]],
                              "passes": 3, "warmup_passes": 1,
                              "sm_mhz_each_pass": [c.get("sm_mhz") if c else None for c in pass_clocks],
                              "drift_pct_clock_normalised_each_pass": drift_norm,
                              # late chunks of a pass against the early chunks of the pass that follows it
                              # (seconds apart, so both run in the same power and clock state of the GPU)
                              "drift_pct_adjacent_passes": [
                                  float((np.median(prev[200:225]) - np.median(nxt[5:30])) / np.median(nxt[5:30])
                                        * 100) for prev, nxt in zip([warm_lat] + runs[:-1], runs)],
                              "drift_pct_clock_normalised": (float(np.median([d["pct"] for d in drift_norm if d]))
                                                             if any(drift_norm) else None),
                              "note": "clock-normalised: per pass, median ms x median SM MHz (NVML every 2 ms) "
                                      "of chunks 200-224 against chunks 5-29"}
    # The same stream paced: each chunk starts after an idle gap on the device of about twice its own
    # time (a one-thread sleep kernel), so the GPU is not held at its power cap; one warm-up pass.
    gap_cycles = 1_300_000
    stream_pass(5, gap_cycles)
    paced = [stream_pass(6 + k, gap_cycles)[0] for k in range(2)]
    pm = np.median(np.stack(paced), axis=0)
    pe, pl = float(np.median(pm[5:30])), float(np.median(pm[200:225]))
    out["long_stream_225_paced"] = {
        "gap_cycles": gap_cycles, "ms_per_chunk_median_5_29": pe, "ms_per_chunk_median_200_224": pl,
        "drift_pct": (pl - pe) / pe * 100.0,
        "drift_pct_each_pass": [float((np.median(p[200:225]) - np.median(p[5:30])) / np.median(p[5:30]) * 100)
                                for p in paced],
        "passes": 2, "warmup_passes": 1}

    # ---- memory-bound kernels (bandwidth, L2 flushed before each rep)
    def bw(fn, nbytes, reps=20):
        ts = []
        for _ in range(reps):
            flush.sum()
            torch.cuda._sleep(200000)  # about 100 us: the host queues the timed call meanwhile
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        t = float(np.median(ts)) * 1e-3
        return {"us": t * 1e6, "gbs": nbytes / t / 1e9, "frac_of_hbm": nbytes / t / 1e9 / peak_gbs}
    # launch + event floor: an empty-work kernel between the same events
    tiny = torch.zeros(4, dtype=torch.int32, device=dev)
    out["event_floor_us"] = float(np.median(_timed(lambda: tiny.zero_(), 50, stream))) * 1e3

    # append: one call with L2 flushed (latency), and a stream of back-to-back
    # appends over 8 distinct source chunks (159 MB, more than L2)
    ringa = cca.KVRing(H, D, L, W, device=dev)
    kk, vv = bf(c1.ring_k[0]), bf(c1.ring_v[0])
    chunk_bytes = 4 * L * H * D * 2
    out["append_720p"] = bw(lambda: ringa.append(kk, vv), chunk_bytes)
    srcs = [(torch.randn((L, H, D), device=dev).to(torch.bfloat16), torch.randn((L, H, D), device=dev).to(
        torch.bfloat16)) for _ in range(8)]
    n_app = 24
    ts = []
    for _ in range(5):
        flush.sum()
        torch.cuda._sleep(400000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n_app):
            ringa.append(*srcs[i % 8])
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e-3 / n_app)
    t = float(np.median(ts))
    out["append_720p_stream"] = {"us_per_call": t * 1e6, "gbs": chunk_bytes / t / 1e9,
                                 "frac_of_hbm": chunk_bytes / t / 1e9 / peak_gbs, "calls": n_app}
    del srcs
    # append bandwidth over chunk sizes (the 720p chunk x 1, 4, 16, 64 tokens), L2 flushed before each call
    sweep_app = {}
    for mult in (1, 4, 16, 64):
        n_tok = L * mult
        rs = cca.KVRing(H, D, n_tok, 1, device=dev)
        ks_ = torch.randn((n_tok, H, D), device=dev, dtype=torch.bfloat16)
        vs_ = torch.randn((n_tok, H, D), device=dev, dtype=torch.bfloat16)
        rs.append(ks_, vs_)  # the sink slot; the timed calls rotate through the window slot
        sweep_app[n_tok] = bw(lambda: rs.append(ks_, vs_), 4 * n_tok * H * D * 2, reps=10)
        del rs, ks_, vs_
    out["sweep_append_chunk_tokens"] = sweep_app

    # latency at the 720p mask-cache size (1620 tokens)
    out["mask_dynamic_720p_us"] = float(np.median(_timed(
        lambda: cca.cca_token_mask_l2(src, edit, prune_quantile=0.7, mask=mask), 50, stream))) * 1e3
    out["mask_fixed_720p_us"] = float(np.median(_timed(
        lambda: cca.cca_token_mask_l2(src, edit, tau=1.0, mask=mask), 50, stream))) * 1e3
    out["compact_720p_us"] = float(np.median(_timed(lambda: cca.cca_compact(mask, idx, n_act), 50, stream))) * 1e3
    out["scatter_720p"] = bw(lambda: cca.cca_scatter(oc, idx, n_act, cache, n_max=L), 2 * n_active * H * D * 2)

    # bandwidth sweeps, L2 flushed before each timed call
    sweep_mask, sweep_comp, sweep_scat = {}, {}, {}
    for lg in range(16, 27, 2):
        n = 1 << lg
        sb = torch.randn((n, 16), device=dev)
        eb = sb + 0.5 * torch.randn((n, 16), device=dev)
        mb = torch.empty(n, dtype=torch.uint8, device=dev)
        sweep_mask[lg] = bw(lambda: cca.cca_token_mask_l2(sb, eb, tau=2.0, mask=mb), n * (2 * 16 * 4 + 1), reps=10)
        del sb, eb
        mc = (torch.rand(n, device=dev) < 0.3).to(torch.uint8)
        ic = torch.empty(n, dtype=torch.int32, device=dev)
        nc = torch.empty(1, dtype=torch.int32, device=dev)
        wc = torch.empty(max(cca.cca_compact_workspace_size(n), 16), dtype=torch.uint8, device=dev)
        cca.cca_compact(mc, ic, nc, workspace=wc)
        torch.cuda.synchronize()
        sweep_comp[lg] = bw(lambda: cca.cca_compact(mc, ic, nc, workspace=wc), n + 4 * int(nc.item()), reps=10)
        del mc, ic, mb
    row = H * D * 2
    for lg in range(10, 19, 2):  # active rows; the cache holds twice as many
        na_rows = 1 << lg
        ocs = torch.randn((na_rows, H * D), device=dev).to(torch.bfloat16)
        cch = torch.zeros((2 * na_rows, H * D), device=dev, dtype=torch.bfloat16)
        ids = torch.arange(0, 2 * na_rows, 2, dtype=torch.int32, device=dev)
        nn = torch.full((1,), na_rows, dtype=torch.int32, device=dev)
        sweep_scat[lg] = bw(lambda: cca.cca_scatter(ocs, ids, nn, cch, n_max=na_rows), 2 * na_rows * row + 4 * na_rows,
                            reps=10)
        del ocs, cch, ids
    out["sweep_mask_fixed_log2_tokens"] = sweep_mask
    out["sweep_compact_log2_tokens"] = sweep_comp
    out["sweep_scatter_log2_active_rows"] = sweep_scat
    out["sweep_note"] = ("bandwidth = algorithmic bytes / event time of one call, L2 flushed before each; append "
                         "2 x 2 x L x H x D bf16 bytes (K and V read and written); mask "
                         "128 B read + 1 B written per token; compaction 1 B read per token + 4 B written per active "
                         "token (30 % active); scatter 2 x 6144 B per active row + 4 B index")
    return out


def extra_rows(dev, stream, peak_tf, peak_gbs):
    """The other hot-path rows at their workload sizes: the clean-pass call, the
    token-group step, the packed block-causal forward, the LiveEdit-shaped chunk,
    the rotary encoding and the e4m3 append.  Inputs are drawn on the device
    (timing only; parity is the tests' job)."""
    import torch
    import chunk_causal_attention_b200 as cca
    out = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    rnd = lambda *sh: torch.randn(*sh, generator=gen, device=dev).to(torch.bfloat16)
    med_us = lambda ts: float(np.median(ts)) * 1e3

    def ring_with(n_tok, window, n_prefill, dtype="bf16"):
        r = cca.KVRing(H, D, n_tok, window, dtype=dtype, device=dev)
        for _ in range(n_prefill):
            r.append(rnd(n_tok, H, D), rnd(n_tok, H, D))
        return r

    # ---- clean pass: the third attention call of a chunk (same shape as a denoising call)
    rings = [ring_with(L, W, 4) for _ in range(3)]
    qkv = [(rnd(L, H, D), rnd(L, H, D), rnd(L, H, D)) for _ in range(3)]
    o = torch.empty((L, H, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(cca.cca_attn_workspace_size(D), dtype=torch.uint8, device=dev)
    it = [0]

    def clean_call():
        i = it[0] % 3
        it[0] += 1
        cca.cca_chunk_attn(rings[i], *qkv[i], out=o, workspace=ws)
    us = med_us(_timed(clean_call, 60, stream))
    out["clean_pass_720p"] = {"us": us, "tflops": FLOP_PER_CALL / (us * 1e-6) / 1e12,
                              "frac_of_bf16_peak": FLOP_PER_CALL / (us * 1e-6) / 1e12 / peak_tf}
    del qkv

    # ---- token groups: N_t (1620) + S_t (1620) + C_t (256) over R (1620), sink + 3 window chunks, themselves
    n_cur, n_ref = L + L + 256, L
    qg, kg, vg = rnd(n_cur, H, D), rnd(n_cur, H, D), rnd(n_cur, H, D)
    kr, vr = rnd(n_ref, H, D), rnd(n_ref, H, D)
    og = torch.empty((n_cur, H, D), dtype=torch.bfloat16, device=dev)
    us = med_us(_timed(lambda: cca.cca_chunk_attn_groups(rings[0], qg, kg, vg, k_ref=kr, v_ref=vr, out=og,
                                                         workspace=ws), 30, stream))
    lk = n_ref + 4 * L + n_cur
    fl = 4.0 * n_cur * lk * H * D
    out["groups_720p"] = {"us": us, "q_tokens": n_cur, "kv_tokens": lk, "tflops": fl / (us * 1e-6) / 1e12,
                          "frac_of_bf16_peak": fl / (us * 1e-6) / 1e12 / peak_tf}
    del qg, kg, vg, kr, vr, og

    # ---- packed block-causal forward: T = 8 chunks of the 720p shape, window 3
    T = 8
    qp, kp, vp, kh, vh = (rnd(T, L, H, D) for _ in range(5))
    op = torch.empty((T, L, H, D), dtype=torch.bfloat16, device=dev)
    us = med_us(_timed(lambda: cca.cca_block_attn(qp, kp, vp, W, k_hist=kh, v_hist=vh, out=op, workspace=ws),
                       10, stream))
    n_vis = sum(1 + (0 if c == 0 else 1 + (c - max(1, c - W))) for c in range(T))
    fl = 4.0 * L * (n_vis * L) * H * D
    out["block_causal_720p_T8"] = {"us": us, "chunks": T, "window": W, "tflops": fl / (us * 1e-6) / 1e12,
                                   "frac_of_bf16_peak": fl / (us * 1e-6) / 1e12 / peak_tf}
    del qp, kp, vp, kh, vh, op

    # ---- LiveEdit-shaped chunk: 3 latent frames (4860 tokens), sink + 2-chunk window, 4 denoising
    # steps on the active tokens of the 3-frame mask (fused scatter-back), the clean pass, the append
    F_, Wl = 3, 2
    Ll = F_ * L
    rl = ring_with(Ll, Wl, 3)
    ql = [rnd(Ll, H, D) for _ in range(4)]
    kl = [rnd(Ll, H, D) for _ in range(4)]
    vl = [rnd(Ll, H, D) for _ in range(4)]
    caches = [rnd(Ll, H, D) for _ in range(4)]
    ol = torch.empty((Ll, H, D), dtype=torch.bfloat16, device=dev)
    src = torch.randn((F_, L, 16), generator=gen, device=dev)
    region = (torch.rand(L, generator=gen, device=dev) < 0.3).float()[None, :, None]
    edit = src + region * (2.0 + torch.randn((F_, L, 16), generator=gen, device=dev)) + \
        (1 - region) * 0.1 * torch.randn((F_, L, 16), generator=gen, device=dev)
    maskl = torch.empty(Ll, dtype=torch.uint8, device=dev)
    idxl = torch.empty(Ll, dtype=torch.int32, device=dev)
    nl = torch.empty(1, dtype=torch.int32, device=dev)

    def liveedit_chunk(append=True):
        cca.cca_token_mask_l2_frames(src, edit, prune_quantile=0.7, mask=maskl)
        cca.cca_compact(maskl, idxl, nl)
        for st in range(4):
            cca.cca_chunk_attn_scatter(rl, ql[st], kl[st], vl[st], idxl, caches[st], n_q_dev=nl, n_q_max=Ll,
                                       workspace=ws)
        cca.cca_chunk_attn(rl, ql[0], kl[0], vl[0], out=ol, workspace=ws)  # clean pass
        if append:
            n0 = rl.n_appended
            rl.append(kl[0], vl[0])
            rl.restore(n0)  # keep the visible set fixed across reps
    ms = float(np.median(_timed(liveedit_chunk, 10, stream)))
    n_act = int(nl.item())
    lkl = (1 + Wl + 1) * Ll
    us_full = med_us(_timed(lambda: cca.cca_chunk_attn(rl, ql[1], kl[1], vl[1], out=ol, workspace=ws), 10, stream))
    us_act = med_us(_timed(lambda: cca.cca_chunk_attn_scatter(rl, ql[1], kl[1], vl[1], idxl, caches[1], n_q_dev=nl,
                                                              n_q_max=Ll, workspace=ws), 10, stream))
    fl_full, fl_act = 4.0 * Ll * lkl * H * D, 4.0 * n_act * lkl * H * D
    out["liveedit_3frame_chunk"] = {
        "ms_per_chunk": ms, "tokens_per_chunk": Ll, "kv_tokens": lkl, "active_tokens": n_act, "steps": 4,
        "full_call_us": us_full, "full_call_tflops": fl_full / (us_full * 1e-6) / 1e12,
        "full_call_frac_of_bf16_peak": fl_full / (us_full * 1e-6) / 1e12 / peak_tf,
        "active_call_us": us_act, "active_call_tflops": fl_act / (us_act * 1e-6) / 1e12,
        "step": "3-frame mask + compaction + 4 active-token attention calls (fused scatter) + clean pass + append"}
    del rl, ql, kl, vl, caches, ol

    # ---- rotary encoding: Q and K of a 720p chunk in one launch; the rotating append
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def bw(fn, nbytes, reps=20):
        ts = []
        for _ in range(reps):
            flush.sum()
            torch.cuda._sleep(200000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        t = float(np.median(ts)) * 1e-3
        return {"us": t * 1e6, "gbs": nbytes / t / 1e9, "frac_of_hbm": nbytes / t / 1e9 / peak_gbs}
    import synth
    pos = torch.from_numpy(synth.grid_positions(4)).to(dev)
    freq = cca.cca_mrope_freqs(D, device=dev)
    qr, kr_ = rnd(L, H, D), rnd(L, H, D)
    qo, ko = torch.empty_like(qr), torch.empty_like(kr_)
    nbytes = 4 * L * H * D * 2
    out["rope_qk_720p"] = bw(lambda: cca.cca_rope_qk(qr, kr_, pos, freq, q_out=qo, k_out=ko), nbytes)
    ra = cca.KVRing(H, D, L, W, device=dev)
    out["append_rope_720p"] = bw(lambda: cca.cca_kv_append_rope(ra, qr, kr_, pos, freq), nbytes)
    r8 = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev)
    e8 = bw(lambda: r8.append(qr, kr_), 2 * L * H * D * 2 + L * H * D + L * H * D * 2)
    e8["note"] = ("algorithmic bytes: read bf16 K and V once (each CTA stages its rows in shared memory for the "
                  "absmax and quantise passes), write K's e4m3 codes and V's codes widened to fp16")
    out["append_e4m3_720p"] = e8
    # the same two kernels over larger token counts (the 720p chunk x 4 and x 16), L2 flushed before each call
    sw_rope, sw_e8 = {}, {}
    for mult in (4, 16):
        n = L * mult
        qn, kn = rnd(n, H, D), rnd(n, H, D)
        qno, kno = torch.empty_like(qn), torch.empty_like(kn)
        posn = pos.repeat((mult,) + (1,) * (pos.dim() - 1))
        sw_rope[n] = bw(lambda: cca.cca_rope_qk(qn, kn, posn, freq, q_out=qno, k_out=kno), 4 * n * H * D * 2,
                        reps=10)
        rn8 = cca.KVRing(H, D, n, 1, dtype="e4m3", device=dev)
        sw_e8[n] = bw(lambda: rn8.append(qn, kn), 2 * n * H * D * 2 + n * H * D + n * H * D * 2, reps=10)
        del qn, kn, qno, kno, rn8
    out["sweep_rope_qk_tokens"] = sw_rope
    out["sweep_append_e4m3_tokens"] = sw_e8
    return out


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import synth
    import chunk_causal_attention_b200 as cca

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.barrier()
    c1 = synth.chunk_720p()
    bf = lambda x: synth.as_torch_bf16(x, dev)

    class Replica:
        def __init__(self):
            self.ring = cca.KVRing(H, D, L, W, device=dev)
            for t in range(c1.t):
                self.ring.append(bf(c1.ring_k[t]), bf(c1.ring_v[t]))
            self.q = [bf(x) for x in c1.q]
            self.k = [bf(x) for x in c1.k_cur]
            self.v = [bf(x) for x in c1.v_cur]
            self.out = [torch.empty((L, H, D), dtype=torch.bfloat16, device=dev) for _ in c1.q]
            ws = cca.cca_chunk_attn_workspace_size(self.ring, L)
            self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)

    reps = [Replica() for _ in range(3)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(rep, ev=None):
        for s in range(CALLS_PER_STEP):
            if ev is not None:
                ev[2 * s].record(stream)
            cca.cca_chunk_attn(rep.ring, rep.q[s], rep.k[s], rep.v[s], out=rep.out[s], workspace=rep.ws)
            if ev is not None:
                ev[2 * s + 1].record(stream)
        rep.ring.append(rep.k[-1], rep.v[-1])  # clean K/V of the chunk (values are immaterial to timing)

    for i in range(args.warmup):
        step(reps[i % 3])
    torch.cuda.synchronize()

    sampler = clock_sampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
    attn_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * CALLS_PER_STEP)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cca.cca_take_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(reps[i % 3], attn_ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = cca.cca_take_launch_count()
    clocks = sampler.stop() if sampler else None
    total_ms = t_start.elapsed_time(t_end)
    attn_ms = [attn_ev[i][2 * s].elapsed_time(attn_ev[i][2 * s + 1]) for i in range(args.steps)
               for s in range(CALLS_PER_STEP)]
    for r in reps:
        torch.cuda.synchronize()
        if int(r.ring.status.item()) != 0:
            raise RuntimeError(f"device status {int(r.ring.status.item())}")
    total_ms = max_over_ranks(total_ms, dev)

    # ---- end to end through the public API with host buffers (pinned), rank-local
    e2e = None
    if args.e2e_steps > 0:
        # Two buffer sets, three streams: the inputs of step k+1 go up (copy
        # engine, s_in) while step k computes (s_c) and step k-1's outputs come
        # down (s_out).  Every step still copies all of its inputs and outputs.
        pin = lambda x: synth.as_torch_bf16(x).pin_memory()
        hq = [pin(x) for x in c1.q]
        hk = [pin(x) for x in c1.k_cur]
        hv = [pin(x) for x in c1.v_cur]
        ho = [[torch.empty((L, H, D), dtype=torch.bfloat16).pin_memory() for _ in c1.q] for _ in range(2)]
        rep = reps[0]
        dq = [[torch.empty_like(x, device=dev) for x in hq] for _ in range(2)]
        dk = [[torch.empty_like(x, device=dev) for x in hk] for _ in range(2)]
        dv = [[torch.empty_like(x, device=dev) for x in hv] for _ in range(2)]
        do = [[torch.empty((L, H, D), dtype=torch.bfloat16, device=dev) for _ in c1.q] for _ in range(2)]
        s_in, s_out, s_c = torch.cuda.Stream(dev), torch.cuda.Stream(dev), stream
        ev = lambda: torch.cuda.Event()
        in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]

        def e2e_step(k):
            b = k & 1
            if used[b]:
                s_in.wait_event(comp_done[b])  # step k-2 no longer reads this input set
            with torch.cuda.stream(s_in):
                for s_ in range(CALLS_PER_STEP):
                    dq[b][s_].copy_(hq[s_], non_blocking=True)
                    dk[b][s_].copy_(hk[s_], non_blocking=True)
                    dv[b][s_].copy_(hv[s_], non_blocking=True)
                in_ready[b].record(s_in)
            s_c.wait_event(in_ready[b])
            if used[b]:
                s_c.wait_event(out_done[b])  # step k-2's outputs have been read back
            for s_ in range(CALLS_PER_STEP):
                cca.cca_chunk_attn(rep.ring, dq[b][s_], dk[b][s_], dv[b][s_], out=do[b][s_], workspace=rep.ws,
                                   stream=s_c)
            rep.ring.append(dk[b][-1], dv[b][-1], stream=s_c)
            comp_done[b].record(s_c)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                for s_ in range(CALLS_PER_STEP):
                    ho[b][s_].copy_(do[b][s_], non_blocking=True)
                out_done[b].record(s_out)
            used[b] = True

        for k in range(3):
            e2e_step(k)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_c)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for k in range(args.e2e_steps):
            e2e_step(k)
        s_c.wait_event(in_ready[(args.e2e_steps - 1) & 1])
        s_c.wait_event(out_done[(args.e2e_steps - 1) & 1])
        e1.record(s_c)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)
        h2d = CALLS_PER_STEP * 3 * L * H * D * 2
        d2h = CALLS_PER_STEP * L * H * D * 2
        e2e = {"value": job_value(world, CALLS_PER_STEP * FLOP_PER_CALL, e2e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    if rank != 0:
        return
    peak_tf, _, peak_kind = peaks()
    ms_step = total_ms / args.steps
    value = job_value(world, CALLS_PER_STEP * FLOP_PER_CALL, ms_step)
    attn_mean_ms = float(np.mean(attn_ms))
    achieved = FLOP_PER_CALL / (attn_mean_ms * 1e-3) / 1e12
    traffic = None
    prof = os.path.join(ROOT, "profiles", "attn_bf16_720p.traffic.json")
    if os.path.exists(prof):
        # counters taken on another build of the kernel do not describe this one
        try:
            import hashlib
            rec = json.load(open(prof))
            src = os.path.join(ROOT, "chunk_causal_attention_b200", "csrc", "attn.cu")
            if rec.get("attn_cu_sha256") == hashlib.sha256(open(src, "rb").read()).hexdigest():
                traffic = rec.get("dram_bytes_per_launch")
        except Exception:
            traffic = None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": world, "seq_len": L, "kv_len": LK, "heads": H,
                   "head_dim": D, "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2: steps cycle 3 replicas (~420 MB)"},
        "ms_per_chunk": ms_step,
        "attn_us_per_call": attn_mean_ms * 1e3,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved / peak_tf, "traffic": traffic,
                     "kernel": "attn_bf16_kernel (+ split-KV combine), per cca_chunk_attn call",
                     "peak_kind": f"bf16 dense, {peak_kind} burst"},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "e2e": e2e,
    }
    if args.extras:
        peak_tf_, peak_gbs_, _ = peaks()
        dev0 = torch.device("cuda", local_rank)
        ex = extra_workloads(dev0, torch.cuda.current_stream(), peak_tf_, peak_gbs_)
        ex.update(extra_rows(dev0, torch.cuda.current_stream(), peak_tf_, peak_gbs_))
        line["rows"] = row_summary(line, ex)
        line["extra"] = ex
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


def row_summary(line, ex):
    """One compact figure per hot-path row, ahead of the long "extra" block."""
    g = lambda *ks: _dig(ex, ks)
    mhz = (line.get("clocks") or {}).get("sm_mhz")
    r = {
        "a1_append_720p_us": g("append_720p", "us"), "a1_append_stream_frac_hbm": g("append_720p_stream", "frac_of_hbm"),
        "a1_append_sweep_103680_tok_frac_hbm": g("sweep_append_chunk_tokens", 103680, "frac_of_hbm"),
        "a2_append_e4m3_720p_us": g("append_e4m3_720p", "us"),
        "a2_append_e4m3_sweep_25920_tok_frac_hbm": g("sweep_append_e4m3_tokens", 25920, "frac_of_hbm"),
        "a3_bf16_call_us": line["attn_us_per_call"], "a3_bf16_frac": line["roofline"]["frac"],
        "a3_bf16_call_us_at_1965mhz": line["attn_us_per_call"] * mhz / 1965.0 if mhz else None,
        "a3_clean_pass_us": g("clean_pass_720p", "us"),
        "a3_fp8_call_us": g("fp8_720p", "attn_us_per_call"), "a3_fp8_frac": g("fp8_720p", "frac_of_fp8_peak"),
        "a4_mask_dynamic_us": g("mask_dynamic_720p_us"), "a4_mask_sweep_2^26_frac_hbm":
            g("sweep_mask_fixed_log2_tokens", 26, "frac_of_hbm"),
        "a5_compact_sweep_2^26_frac_hbm": g("sweep_compact_log2_tokens", 26, "frac_of_hbm"),
        "a6_active_486_attn_us": g("mask_cached_720p", "attn_us"),
        "a7_scatter_sweep_2^18_frac_hbm": g("sweep_scatter_log2_active_rows", 18, "frac_of_hbm"),
        "c2_drift_pct": g("long_stream_225", "drift_pct"),
        "c2_drift_pct_clock_normalised": g("long_stream_225", "drift_pct_clock_normalised"),
        "c2_drift_pct_paced": g("long_stream_225_paced", "drift_pct"),
        "c2_drift_pct_adjacent_passes_median": (float(np.median(ex["long_stream_225"]["drift_pct_adjacent_passes"]))
                                                 if "long_stream_225" in ex else None),
        "f1_groups_us": g("groups_720p", "us"), "f1_groups_frac": g("groups_720p", "frac_of_bf16_peak"),
        "f2_rope_qk_frac_hbm": g("rope_qk_720p", "frac_of_hbm"),
        "f2_rope_qk_sweep_25920_tok_frac_hbm": g("sweep_rope_qk_tokens", 25920, "frac_of_hbm"),
        "f2_append_rope_frac_hbm": g("append_rope_720p", "frac_of_hbm"),
        "f3_liveedit_ms_per_chunk": g("liveedit_3frame_chunk", "ms_per_chunk"),
        "f3_liveedit_full_call_frac": g("liveedit_3frame_chunk", "full_call_frac_of_bf16_peak"),
        "f4_block_T8_us": g("block_causal_720p_T8", "us"),
        "f4_block_T8_frac": g("block_causal_720p_T8", "frac_of_bf16_peak"),
    }
    return r


def _dig(d, ks):
    for k in ks:
        if not isinstance(d, dict):
            return None
        d = d.get(k, d.get(str(k)))
    return d


# ------------------------------------------------------------------ profiling cases
def profile_case(name: str) -> None:
    """Run one kernel a few times on its workload (L2 flushed in between) and
    exit: a small, self-contained target for ncu captures."""
    import torch
    import chunk_causal_attention_b200 as cca
    dev = torch.device("cuda:0")
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    if name == "compact_64M":
        n = 1 << 26
        mc = (torch.rand(n, device=dev) < 0.3).to(torch.uint8)
        idx = torch.empty(n, dtype=torch.int32, device=dev)
        na = torch.empty(1, dtype=torch.int32, device=dev)
        ws = torch.empty(cca.cca_compact_workspace_size(n), dtype=torch.uint8, device=dev)
        fn = lambda: cca.cca_compact(mc, idx, na, workspace=ws)
    elif name == "append_720p":
        ring = cca.KVRing(H, D, L, W, device=dev)
        k = torch.randn((L, H, D), device=dev).to(torch.bfloat16)
        v = torch.randn((L, H, D), device=dev).to(torch.bfloat16)
        fn = lambda: ring.append(k, v)
    elif name == "mask_fixed_16M":
        n = 1 << 24
        src = torch.randn((n, 16), device=dev)
        edit = src + 0.5 * torch.randn((n, 16), device=dev)
        mask = torch.empty(n, dtype=torch.uint8, device=dev)
        fn = lambda: cca.cca_token_mask_l2(src, edit, tau=2.0, mask=mask)
    elif name == "scatter_64K_rows":
        n = 1 << 16
        oc = torch.randn((n, H * D), device=dev).to(torch.bfloat16)
        cache = torch.zeros((2 * n, H * D), device=dev, dtype=torch.bfloat16)
        ids = torch.arange(0, 2 * n, 2, dtype=torch.int32, device=dev)
        nn = torch.full((1,), n, dtype=torch.int32, device=dev)
        fn = lambda: cca.cca_scatter(oc, ids, nn, cache)
    elif name == "fp8_720p":
        import synth
        bf = lambda x: synth.as_torch_bf16(x, dev)
        s3 = synth.fp8_720p(n_steps=1)
        ring8 = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev)
        for t in range(s3.t):
            ring8.append(bf(s3.ring_k[t]), bf(s3.ring_v[t]))
        q8, qs = cca.cca_quant_e4m3(bf(s3.q[0]))
        k8, ks = cca.cca_quant_e4m3(bf(s3.k_cur[0]))
        v8, vs = cca.cca_quant_e4m3_f16(bf(s3.v_cur[0]))
        ws8 = torch.empty(max(cca.cca_chunk_attn_workspace_size(ring8, L), 16), dtype=torch.uint8, device=dev)
        fn = lambda: cca.cca_chunk_attn(ring8, q8, k8, v8, q_scale=qs, kcur_scale=ks, vcur_scale=vs, workspace=ws8)
    elif name == "masked_720p":
        import synth
        bf = lambda x: synth.as_torch_bf16(x, dev)
        c1 = synth.chunk_720p(n_steps=1)
        m = synth.mask_chunk()
        ring = cca.KVRing(H, D, L, W, device=dev)
        for t in range(c1.t):
            ring.append(bf(c1.ring_k[t]), bf(c1.ring_v[t]))
        mask = cca.cca_token_mask_l2(torch.from_numpy(m.src).to(dev), torch.from_numpy(m.edit).to(dev),
                                     prune_quantile=m.prune_quantile)
        idx, n_act = cca.cca_compact(mask)
        q, kc, vc = bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0])
        wsm = torch.empty(max(cca.cca_chunk_attn_workspace_size(ring, L), 16), dtype=torch.uint8, device=dev)
        fn = lambda: cca.cca_chunk_attn(ring, q, kc, vc, q_idx=idx, n_q_dev=n_act, n_q_max=L, workspace=wsm)
    elif name == "bf16_720p":
        ring = cca.KVRing(H, D, L, W, device=dev)
        for _ in range(4):
            ring.append(torch.randn((L, H, D), device=dev).to(torch.bfloat16),
                        torch.randn((L, H, D), device=dev).to(torch.bfloat16))
        q, kc, vc = (torch.randn((L, H, D), device=dev).to(torch.bfloat16) for _ in range(3))
        ws = torch.empty(cca.cca_chunk_attn_workspace_size(ring, L), dtype=torch.uint8, device=dev)
        fn = lambda: cca.cca_chunk_attn(ring, q, kc, vc, workspace=ws)
    elif name == "mask_select_32K":
        n = 32768
        src = torch.randn((n, 16), device=dev)
        edit = src + 0.5 * torch.randn((n, 16), device=dev)
        mask = torch.empty(n, dtype=torch.uint8, device=dev)
        fn = lambda: cca.cca_token_mask_l2(src, edit, prune_quantile=0.7, mask=mask)
    elif name == "rope_qk_720p":
        import synth
        pos = torch.from_numpy(synth.grid_positions(4)).to(dev)
        freq = cca.cca_mrope_freqs(D, device=dev)
        q, k = (torch.randn((L, H, D), device=dev).to(torch.bfloat16) for _ in range(2))
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        fn = lambda: cca.cca_rope_qk(q, k, pos, freq, q_out=qo, k_out=ko)
    elif name == "append_e4m3_720p":
        ring = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev)
        k = torch.randn((L, H, D), device=dev).to(torch.bfloat16)
        v = torch.randn((L, H, D), device=dev).to(torch.bfloat16)
        fn = lambda: ring.append(k, v)
    else:
        raise SystemExit(f"unknown profile case {name}")
    for _ in range(3):
        flush.sum()
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extras", type=int, default=1, help="also time the fp8, mask-cached, long-stream and "
                    "memory-bound workloads (rank 0, extra keys)")
    ap.add_argument("--profile-case", default=None,
                    help="only run one kernel three times, for ncu: compact_64M, append_720p, mask_fixed_16M, "
                    "scatter_64K_rows, fp8_720p (e4m3 attention), masked_720p (486 gathered queries)")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
