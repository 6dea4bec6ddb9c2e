#!/usr/bin/env python
"""Throughput of the GigaAM Conformer encoder + CTC path on B200.

One step = gam_encode + gam_ctc_greedy over one batch of a synthetic workload
(audio already resident in device memory).  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (launched by torchrun, one process per GPU): every rank runs its own
copy of the workload batch (independent clips, no data-path collective), the
elapsed time is the max over ranks, value = total audio seconds / that time
(weak scaling).

``--impl reference`` times the CPU oracle (the plain NumPy definition of the
path) on this machine's host cores, one bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from conformer_speech_recognition_b200 import synth  # noqa: E402

METRIC = "audio-sec/sec (×realtime) encoder+CTC at 1 B200; GEMM TFLOP/s vs fp16 peak"
UNIT = "audio-sec/sec"
# The largest configuration that runs on one GPU: 32 x 30 s clips on the 24-layer
# d1024 encoder (about 30 TFLOP per step).
DEFAULT_WORKLOAD = "c4_30s_b32_d1024"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def fp16_vs_bf16_matmul(device, n=8192, iters=10):
    """Library (cuBLAS) dense matmul rate in fp16 and bf16 on this GPU, n^3 shape,
    best of `iters` with CUDA events: a check that the fp16 tensor-core peak the
    roofline uses equals the measured bf16 one.  Not part of the timed path."""
    import torch
    out = {}
    for name, dt in (("fp16", torch.float16), ("bf16", torch.bfloat16)):
        a = torch.randn(n, n, device=device, dtype=dt)
        b = torch.randn(n, n, device=device, dtype=dt)
        for _ in range(3):
            torch.matmul(a, b)
        best = float("inf")
        for _ in range(iters):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b)
            e1.record()
            torch.cuda.synchronize(device)
            best = min(best, e0.elapsed_time(e1))
        out[name + "_tflops"] = 2.0 * n ** 3 / (best / 1e3) / 1e12
        del a, b
    out["fp16_over_bf16"] = out["fp16_tflops"] / out["bf16_tflops"]
    return out


def pick_peak(peaks, clocks):
    """The tensor peak (measured, else the fallback) that applies to this run: the burst figure when
    the SM clock sampled during the timed region sat within 3% of its maximum
    (no power-cap throttling), else the sustained figure (measured under the
    power cap).  Returns (peak TFLOP/s, "burst" | "sustained")."""
    sm, smax = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    if sm and smax and sm >= 0.97 * smax:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


# Dense fp16 tensor-core work per SM per clock on sm_100 (4096 FMA), for the
# nominal peak at the sampled clock reported beside the measured one.
FP16_FLOP_PER_SM_CLK = 8192


def roofline_object(dominant, fl, by, dom_ms, dom_n, steps, peaks, clocks, workload, sms=148):
    """Roofline of the dominant kernel family over the timed region: algorithmic
    work per launch / mean launch time, against the measured peak that applies."""
    avg_launch_ms = dom_ms / max(dom_n, 1)
    launches_per_step = dom_n / steps
    if dominant in fl and dominant != "frontend":
        per_launch = fl[dominant] / launches_per_step
        achieved = per_launch / (avg_launch_ms / 1e3) / 1e12
        peak, kind = pick_peak(peaks, clocks)
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": measured_traffic(workload, dominant), "kernel": dominant,
                "flop_per_launch": per_launch, "launches_per_step": launches_per_step,
                "mean_launch_ms": avg_launch_ms,
                "peak_source": f"{peaks['source']} bf16 dense {kind} (fp16 = bf16 rate on sm_100; "
                               f"median SM clock {((clocks or {}).get('sm_mhz'))} of max "
                               f"{((clocks or {}).get('sm_max_mhz'))} MHz)",
                "frac_vs_burst": achieved / peaks["bf16_tflops"],
                "frac_vs_sustained": achieved / peaks["bf16_tflops_sustained"]}
        sm = (clocks or {}).get("sm_mhz")
        if sm:
            nominal = FP16_FLOP_PER_SM_CLK * sms * sm * 1e6 / 1e12
            roof["nominal_fp16_at_sampled_clock_tflops"] = nominal
            roof["frac_vs_nominal_at_sampled_clock"] = achieved / nominal
        return roof
    per_launch = by.get(dominant, 0.0) / max(launches_per_step, 1)
    achieved = per_launch / (avg_launch_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": measured_traffic(workload, dominant), "kernel": dominant, "bytes_per_launch": per_launch,
            "mean_launch_ms": avg_launch_ms, "peak_source": f"{peaks['source']} HBM copy"}


def algorithmic_work(cfg, lens):
    """Per-kernel-family algorithmic FLOPs or bytes for ONE step, and the number of
    launches of each family per step.  Valid frames only (padding excluded)."""
    from conformer_speech_recognition_b200 import gam
    fr, el, fmax, tmax = gam.gam_plan_lengths(cfg, lens)
    d, f, L, C = cfg["d_model"], cfg["ffn_dim"], cfg["n_layers"], cfg["n_classes"]
    Kdw = cfg["conv_kernel"]
    M = float(np.sum(el))
    L1 = float(np.sum((fr - 1) // 2))
    att = float(np.sum(el.astype(np.float64) ** 2))
    wbytes = 1 if cfg["precision"] == "int8_g64" else 2
    act = 2  # fp16 activations
    fl = {
        "gemm_subsampling": 2 * L1 * 5 * cfg["n_mels"] * d + 2 * M * 5 * d * d,
        "gemm_ffn_up": 2 * L * 2 * M * d * f,
        "gemm_ffn_down": 2 * L * 2 * M * f * d,
        "gemm_qkv": L * 2 * M * d * 3 * d,
        "gemm_attn_out": L * 2 * M * d * d,
        "gemm_pw1_glu": L * 2 * M * d * 2 * d,
        "gemm_pw2": L * 2 * M * d * d,
        "attention": L * 4 * att * d,
        "ctc_gemm": 2 * M * d * C,
        "frontend": float(np.sum(fr)) * (2 * 320 * 320 + 2 * 161 * 64),
    }
    by = {
        "layernorm": L * 5 * M * d * (4 + act),
        "dwconv": L * M * d * 2 * act,
        "frontend": float(np.sum(lens)) * 4 + float(np.sum(fr)) * 64 * act,
    }
    launches = {"gemm_subsampling": 2, "gemm_ffn_up": 2 * L, "gemm_ffn_down": 2 * L, "gemm_qkv": L,
                "gemm_attn_out": L, "gemm_pw1_glu": L, "gemm_pw2": L, "attention": L, "ctc_gemm": 1,
                "frontend": 1, "layernorm": 4 * L + 1, "dwconv": L}
    _ = wbytes
    return fl, by, launches


def measured_traffic(workload, family):
    """DRAM bytes per launch of `family` from the committed ncu summary
    (profiles/traffic.json), or None when there is none for this workload or the
    kernel source changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[workload][family]
        src = os.path.join(ROOT, entry["kernel_source"])
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != entry["kernel_source_sha256_16"]:
                return None
        return entry["bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


def time_workload(name, steps=5, warmup=3, weights=None, device=0, peaks=None, clocks=None):
    """×realtime of one workload on this GPU: gam_encode + gam_ctc_greedy with the
    audio resident, CUDA events over `steps` steps after `warmup` steps (CUDA
    graphs on).  Then `steps` more steps with the dominant kernel family timed by
    events around each launch give its roofline object."""
    import torch
    from conformer_speech_recognition_b200 import gam
    cfg = synth.workload_config(name)
    W = weights if weights is not None else synth.random_weights(cfg, seed=0)
    audio_np, lens = synth.workload_audio(name)
    B, nmax = audio_np.shape
    ctx = gam.gam_create(cfg, W, B, nmax, device=device)
    try:
        dev = torch.device("cuda", device)
        audio = torch.from_numpy(audio_np).to(dev)
        _, el, _, tmax = gam.gam_plan_lengths(cfg, lens)
        enc = torch.empty((B, tmax, cfg["d_model"]), dtype=torch.float32, device=dev)
        tok = torch.empty((B, tmax), dtype=torch.int32, device=dev)
        cnt = torch.empty((B,), dtype=torch.int32, device=dev)
        stream = torch.cuda.current_stream(dev)

        def step():
            gam.gam_encode(ctx, audio, lens, out=enc, stream=stream)
            gam.gam_ctc_greedy(ctx, enc, el, stream=stream, tokens=tok, counts=cnt)

        for _ in range(warmup):
            step()
        torch.cuda.synchronize(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        ms = t0.elapsed_time(t1) / steps
        audio_s = float(np.sum(lens)) / synth.SAMPLE_RATE
        out = {"value": audio_s / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps, "warmup": warmup,
               "batch": int(B), "audio_seconds_per_step": audio_s, "precision": cfg["precision"]}
        if peaks is not None:
            gam.gam_profile_enable(ctx, -1)
            step()
            torch.cuda.synchronize(dev)
            warm = gam.gam_profile_all(ctx)
            dominant = max(warm, key=lambda n: warm[n][0])
            kinds = {gam.gam_profile_kind_name(k): k for k in range(gam.gam_profile_kinds())}
            gam.gam_profile_enable(ctx, 1 << kinds[dominant])
            for _ in range(steps):
                step()
            torch.cuda.synchronize(dev)
            dom_ms, dom_n = gam.gam_profile_read(ctx, kinds[dominant])
            fl, by, _ = algorithmic_work(cfg, lens)
            out["roofline"] = roofline_object(dominant, fl, by, dom_ms, dom_n, steps, peaks, clocks, name)
            out["profile_ms_per_step"] = {k: round(v[0], 4) for k, v in warm.items() if v[1]}
            gam.gam_profile_enable(ctx, 0)
        return out
    finally:
        ctx.close()


def time_rnnt(name, n_classes, steps=5, warmup=3, weights=None, device=0):
    """Encoder + greedy RNNT decoding of a workload's batch (audio resident): the
    whole step, and the decoder part (joint encoder projection + sequential
    decode) alone, with CUDA events."""
    import torch
    from conformer_speech_recognition_b200 import gam
    cfg = synth.workload_config(name)
    W = weights if weights is not None else synth.random_weights(cfg, seed=0)
    audio_np, lens = synth.workload_audio(name)
    B, nmax = audio_np.shape
    ctx = gam.gam_create(cfg, W, B, nmax, device=device)
    try:
        dev = torch.device("cuda", device)
        # the synthetic encoder output is strongly correlated from frame to frame, so the
        # blank offset that gives a speech-like symbol rate depends on the class count
        blank_bias = {34: 3.0, 1025: 5.0}.get(n_classes, 7.0)
        gam.gam_rnnt_attach(ctx, dict(synth.RNNT, n_classes=n_classes),
                            synth.random_rnnt_weights(cfg["d_model"], n_classes, blank_bias=blank_bias))
        audio = torch.from_numpy(audio_np).to(dev)
        _, el, _, tmax = gam.gam_plan_lengths(cfg, lens)
        enc = torch.empty((B, tmax, cfg["d_model"]), dtype=torch.float32, device=dev)
        mt = tmax * synth.RNNT["max_symbols"]
        tok = torch.empty((B, mt), dtype=torch.int32, device=dev)
        frm = torch.empty((B, mt), dtype=torch.int32, device=dev)
        cnt = torch.empty((B,), dtype=torch.int32, device=dev)
        stream = torch.cuda.current_stream(dev)

        def dec():
            gam.gam_rnnt_greedy(ctx, enc, el, max_tokens=mt, stream=stream, tokens=tok, frames=frm, counts=cnt)

        def step():
            gam.gam_encode(ctx, audio, lens, out=enc, stream=stream)
            dec()

        for _ in range(warmup):
            step()
        torch.cuda.synchronize(dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        for _ in range(steps):
            step()
        ev[1].record(stream)
        for _ in range(steps):
            dec()
        ev[2].record(stream)
        torch.cuda.synchronize(dev)
        ms = ev[0].elapsed_time(ev[1]) / steps
        dec_ms = ev[1].elapsed_time(ev[2]) / steps
        gam.gam_profile_enable(ctx, -1)
        dec()
        torch.cuda.synchronize(dev)
        prof = gam.gam_profile_all(ctx)
        gam.gam_profile_enable(ctx, 0)
        audio_s = float(np.sum(lens)) / synth.SAMPLE_RATE
        symbols = cnt.cpu().numpy()
        # the clips decode in parallel, one CTA each: the clip with the most decisions
        # (frames + emitted symbols) sets the kernel's time
        decisions = np.asarray(el, np.int64) + symbols.astype(np.int64)
        worst = int(np.argmax(decisions))
        return {"value": audio_s / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "decode_ms": dec_ms,
                "slowest_clip": {"frames": int(el[worst]), "symbols": int(symbols[worst]),
                                 "us_per_decision": prof["rnnt_decode"][0] * 1e3 / max(int(decisions[worst]), 1)},
                "decode_share": dec_ms / ms, "n_classes": n_classes, "steps": steps, "batch": int(B),
                "symbols_per_clip_mean": float(symbols.mean()), "valid_frames": int(np.sum(el)),
                "symbols_per_frame": float(symbols.sum()) / max(int(np.sum(el)), 1), "blank_bias": blank_bias,
                "rnnt_enc_proj_ms": prof["rnnt_enc_proj"][0], "rnnt_decode_kernel_ms": prof["rnnt_decode"][0],
                "audio_seconds_per_step": audio_s}
    finally:
        ctx.close()


def time_streaming(window_s=30.0, push_s=1.0, total_s=60.0, weights=None, device=0):
    """Pseudo-streaming on the v3 d768 model: pushes of push_s seconds of audio
    for total_s seconds, every push re-recognising the last window_s seconds.
    Reports audio pushed per second of wall time and the per-push latency once
    the window is full (host-timed: each push synchronises)."""
    import torch
    from conformer_speech_recognition_b200 import gam
    cfg = synth.workload_config("c1_1s_b1_d768")
    W = weights if weights is not None else synth.random_weights(cfg, seed=0)
    win = int(window_s * synth.SAMPLE_RATE)
    ctx = gam.gam_create(cfg, W, 1, win, device=device)
    try:
        st = gam.Stream(ctx, win)
        x, _ = synth.random_audio([int(total_s * synth.SAMPLE_RATE)], seed=55)
        x = x[0]
        n = int(push_s * synth.SAMPLE_RATE)
        for k in range(3):  # warm-up pushes (graphs are captured on the window's second sighting)
            st.push(x[k * n:(k + 1) * n])
        st.reset()
        torch.cuda.synchronize(device)
        lat = []
        t_all = time.perf_counter()
        for k in range(0, len(x) // n):
            t0 = time.perf_counter()
            st.push(x[k * n:(k + 1) * n])
            lat.append(time.perf_counter() - t0)
        wall = time.perf_counter() - t_all
        full = lat[int(window_s / push_s) + 2:]
        st.close()
        return {"value": total_s / wall, "unit": UNIT, "window_s": window_s, "push_s": push_s,
                "pushes": len(lat), "latency_ms_full_window_median": 1e3 * statistics.median(full) if full else None,
                "latency_ms_first_push": 1e3 * lat[0]}
    finally:
        ctx.close()


def chunk_sweep(device=0, steps=3):
    """The pages' long-form shape question ("GigaAM MLX port for Mac",
    "Which optimizations actually made the model faster": 20 s vs 40 s chunks,
    groups of 8): the 300 s chirp on the d1024 model as 15 x 20 s or 8 x 40 s
    chunks, all in one batch or in groups of 8, with fp16, INT8, INT6 and INT4
    weights; then the batch size (1 to 64 clips of 20 s) on the d1024 model."""
    import torch
    from conformer_speech_recognition_b200 import gam
    full, _ = synth.workload_audio("c5_300s_chunks15_d1024_int8")
    x = full.reshape(-1)
    out = {}
    for prec in ("fp16", "int8_g64", "int6_g64", "int4_g64"):
        cfg = synth.model_config(synth.LARGE, 257, prec)
        W = synth.random_weights(cfg, seed=0)
        ctx = gam.gam_create(cfg, W, 15, 40 * synth.SAMPLE_RATE, device=device)
        try:
            for chunk_s in (20, 40):
                c = chunk_s * synth.SAMPLE_RATE
                n = (len(x) + c - 1) // c
                audio = np.zeros((n, c), np.float32)
                lens = np.zeros(n, np.int32)
                for k in range(n):
                    seg = x[k * c:(k + 1) * c]
                    audio[k, :len(seg)] = seg
                    lens[k] = len(seg)
                a = torch.from_numpy(audio).cuda(device)
                for group in (n, 8):
                    calls = [(i, min(i + group, n)) for i in range(0, n, group)]

                    def step():
                        for i0, i1 in calls:
                            enc, el = gam.gam_encode(ctx, a[i0:i1], lens[i0:i1])
                            gam.gam_ctc_greedy(ctx, enc, el)
                    for _ in range(2):
                        step()
                    torch.cuda.synchronize(device)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    for _ in range(steps):
                        step()
                    e1.record()
                    torch.cuda.synchronize(device)
                    ms = e0.elapsed_time(e1) / steps
                    out[f"{prec}_{chunk_s}s_x{n}_groups_of_{group}"] = {"value": (len(x) / synth.SAMPLE_RATE) / (ms / 1e3),
                                                                       "unit": UNIT, "ms": ms}
        finally:
            ctx.close()
    # batch size for throughput: B clips of 20 s (the C3 clip recipe) on the d1024 model, fp16
    cfg = synth.model_config(synth.LARGE, 257, "fp16")
    W = synth.random_weights(cfg, seed=0)
    audio64, lens64 = synth.workload_audio("c3_20s_b64_d768")
    ctx = gam.gam_create(cfg, W, 64, int(lens64.max()), device=device)
    try:
        for B in (1, 4, 8, 16, 32, 64):
            a = torch.from_numpy(np.ascontiguousarray(audio64[:B])).cuda(device)
            ln = lens64[:B]

            def step():
                enc, el = gam.gam_encode(ctx, a, ln)
                gam.gam_ctc_greedy(ctx, enc, el)
            for _ in range(2):
                step()
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                step()
            e1.record()
            torch.cuda.synchronize(device)
            ms = e0.elapsed_time(e1) / steps
            out[f"fp16_d1024_20s_batch_{B}"] = {"value": float(np.sum(ln)) / synth.SAMPLE_RATE / (ms / 1e3),
                                                "unit": UNIT, "ms": ms}
    finally:
        ctx.close()
    return out


def reduce_max_over_ranks(values, device=None):
    """Element-wise max over all ranks (torch.distributed all_reduce MAX)."""
    import torch
    import torch.distributed as td
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, audio_seconds_per_rank_step, steps, elapsed_ms):
    """Whole-job audio-s/s: every rank processed its own batch each step; the job
    took the slowest rank's time."""
    return world * audio_seconds_per_rank_step * steps / (elapsed_ms / 1e3)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_throughput(name, budget_s, clip_indices=None):
    """The CPU oracle (fp32, as it stands) on a bounded sample of the workload.
    Returns (audio seconds per second, description, threads)."""
    import oracle
    cfg = synth.workload_config(name)
    W = synth.random_weights(cfg, seed=0)
    audio, lens = synth.workload_audio(name)
    order = clip_indices if clip_indices is not None else list(range(len(lens)))
    done_audio = 0.0
    used = []
    t0 = time.perf_counter()
    for i in order:
        oracle.transcribe_clip(audio[i, :lens[i]], W, cfg, np.float32)
        done_audio += lens[i] / synth.SAMPLE_RATE
        used.append(int(i))
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    desc = f"{len(used)} clip(s) {used[:8]}{'...' if len(used) > 8 else ''} of {name}, {done_audio:.1f} audio-s, " \
           f"fp32 NumPy oracle, {el:.1f} s"
    return done_audio / el, desc, threads


# ---------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    name = args.workload
    cfg = synth.workload_config(name)
    import oracle
    W = synth.random_weights(cfg, seed=0)
    audio, lens = synth.workload_audio(name)
    order = list(np.argsort(lens))  # shortest clips first keeps every step bounded
    cap = int(args.ref_seconds * synth.SAMPLE_RATE)
    per_step = []
    audio_s = []

    def one(i):
        n = int(min(lens[i], cap))
        t0 = time.perf_counter()
        oracle.transcribe_clip(audio[i, :n], W, cfg, np.float32)
        return time.perf_counter() - t0, n / synth.SAMPLE_RATE

    k = 0
    for _ in range(args.warmup):
        one(order[k % len(order)])
        k += 1
    for _ in range(args.steps):
        t, a = one(order[k % len(order)])
        per_step.append(t)
        audio_s.append(a)
        k += 1
    total_t, total_a = sum(per_step), sum(audio_s)
    value = total_a / total_t
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    sample = (f"one clip per step (shortest first, cut to at most {args.ref_seconds:g} s) of {name}: "
              f"{total_a:.1f} audio-s over {args.steps} steps")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": name, "batch": 1, "precision": "fp32 oracle (NumPy)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    from conformer_speech_recognition_b200 import gam
    dist = world > 1
    if dist:
        import torch.distributed as td
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    name = args.workload
    cfg = synth.workload_config(name)
    W = synth.random_weights(cfg, seed=0)
    audio_np, lens = synth.workload_audio(name)
    B, nmax = audio_np.shape
    ctx = gam.gam_create(cfg, W, B, nmax, device=local_rank)
    audio = torch.from_numpy(audio_np).to(dev)
    fr, el, fmax, tmax = gam.gam_plan_lengths(cfg, lens)
    enc = torch.empty((B, tmax, cfg["d_model"]), dtype=torch.float32, device=dev)
    tok = torch.empty((B, tmax), dtype=torch.int32, device=dev)
    cnt = torch.empty((B,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    audio_seconds = float(np.sum(lens)) / synth.SAMPLE_RATE

    def step():
        gam.gam_encode(ctx, audio, lens, out=enc, stream=stream)
        return gam.gam_ctc_greedy(ctx, enc, el, stream=stream, tokens=tok, counts=cnt)

    # warm-up (untimed), then two profiled steps with every kernel family timed:
    # the per-family table and the dominant family come from steady-state steps
    gam.gam_profile_enable(ctx, 0)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    gam.gam_profile_enable(ctx, -1)
    n_prof = 2
    for _ in range(n_prof):
        step()
    torch.cuda.synchronize(dev)
    warm = gam.gam_profile_all(ctx)
    kinds = {gam.gam_profile_kind_name(k): k for k in range(gam.gam_profile_kinds())}
    dominant = max(warm, key=lambda n: warm[n][0])

    # timed region: only the dominant family carries event pairs
    gam.gam_profile_enable(ctx, 1 << kinds[dominant])
    clocks = ClockSampler(local_rank) if rank == 0 else None
    if dist:
        td.barrier()
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    elapsed_ms = t_start.elapsed_time(t_end)
    clock_info = clocks.stop() if clocks else None
    prof = gam.gam_profile_all(ctx)
    launches = sum(v[1] for v in prof.values())
    dom_ms, dom_n = prof[dominant]
    gam.gam_device_status(ctx)

    # end to end through the public host-buffer call (copies inside the timed region)
    pinned = torch.from_numpy(audio_np).pin_memory()
    tok_h = torch.empty((B, tmax), dtype=torch.int32).pin_memory()
    cnt_h = torch.empty((B,), dtype=torch.int32).pin_memory()
    gam.gam_profile_enable(ctx, 0)
    for _ in range(max(1, args.warmup)):
        gam.gam_transcribe(ctx, pinned, lens, tok_h, cnt_h, stream=stream)
    if dist:
        td.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        gam.gam_transcribe(ctx, pinned, lens, tok_h, cnt_h, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)

    if dist:
        elapsed_ms, e2e_ms = reduce_max_over_ranks([elapsed_ms, e2e_ms], device=dev)

    if rank == 0:
        peaks = load_peaks()
        fl, by, _ = algorithmic_work(cfg, lens)
        value = job_throughput(world, audio_seconds, args.steps, elapsed_ms)
        e2e_value = job_throughput(world, audio_seconds, args.steps, e2e_ms)
        roof = roofline_object(dominant, fl, by, dom_ms, dom_n, args.steps, peaks, clock_info, name)
        peak_check = fp16_vs_bf16_matmul(dev) if world == 1 else None
        gemm_flops = sum(v for k, v in fl.items() if k.startswith("gemm_"))
        # GEMM kernel time per step from the profiled steps (every family timed there)
        gemm_ms = sum(v[0] for k, v in warm.items() if k.startswith("gemm_")) / n_prof
        gemm_rate = gemm_flops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
        tensor_peak, peak_kind = pick_peak(peaks, clock_info)
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            v, desc, threads = oracle_throughput(name, args.cpu_budget)
            cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}
        per_workload = None
        if world == 1 and not args.no_per_workload:
            per_workload = {}
            for other in sorted(synth.WORKLOADS):
                if other == name:
                    continue
                same_model = synth.workload_config(other) == cfg
                per_workload[other] = time_workload(other, weights=W if same_model else None, device=local_rank,
                                                    peaks=peaks, clocks=clock_info)
        rnnt = stream_res = sweep = None
        if world == 1 and not args.no_per_workload:
            v3 = synth.workload_config("c2_varlen_b32_d768")
            W3 = W if v3 == cfg else None
            rnnt = {"c2_varlen_b32_d768_rnnt34": time_rnnt("c2_varlen_b32_d768", 34, weights=W3, device=local_rank),
                    "c2_varlen_b32_d768_rnnt1025": time_rnnt("c2_varlen_b32_d768", 1025, weights=W3,
                                                             device=local_rank)}
            stream_res = time_streaming(device=local_rank)
        if world == 1 and args.sweep:
            sweep = chunk_sweep(device=local_rank)
        h2d = int(B * nmax * 4 + 5 * (B + 1) * 4 + B * 4)
        d2h = int(B * tmax * 4 + B * 4)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": name, "batch": B, "audio_seconds_per_step": audio_seconds,
                       "valid_encoder_frames": int(np.sum(el)), "precision": cfg["precision"],
                       "layers": cfg["n_layers"], "d_model": cfg["d_model"],
                       "l2": "not flushed: the weights and activations of a step are larger than the 126 MB L2 "
                             "(fp16 weights alone 442 MB at d768, 1.17 GB at d1024)",
                       "parallelism": f"replicas x{world} (independent batches, no collective on the data path)"},
            "roofline": roof,
            "gemm_tflops_per_step_algorithmic": gemm_flops / 1e12,
            "gemm_tflops_per_s_of_gemm_time": gemm_rate,
            "gemm_frac_of_fp16_peak": gemm_rate / tensor_peak if gemm_rate else None,
            "gemm_frac_peak_kind": f"{peaks['source']} bf16 dense {peak_kind} (median SM clock vs max decides)",
            "gemm_frac_of_library_fp16_this_run": gemm_rate / peak_check["fp16_tflops"]
            if gemm_rate and peak_check else None,
            "fp16_peak_check": peak_check,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "clocks": clock_info,
            "profile_ms_per_step": {k: round(v[0] / n_prof, 4) for k, v in warm.items() if v[1]},
            "per_workload": per_workload,
            "rnnt": rnnt,
            "streaming": stream_res,
            "chunk_sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    ctx.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true", help="skip the ×realtime of the other workloads")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU time for cpu_baseline")
    ap.add_argument("--sweep", action="store_true",
                    help="also time the long-form chunk / batch shapes (20 s vs 40 s chunks, groups of 8)")
    ap.add_argument("--ref-seconds", type=float, default=6.0,
                    help="reference arm: each step runs the oracle on one clip cut to at most this many seconds")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: at least 3 warm-up steps are required for a valid number", file=sys.stderr)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch.distributed as td
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as td
            td.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
