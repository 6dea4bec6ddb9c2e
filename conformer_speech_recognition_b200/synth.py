"""Seeded synthetic inputs for the GigaAM Conformer encoder + CTC path.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It only *draws* inputs: audio, clip lengths, model configurations
and named weight tensors in PyTorch layout.  It holds none of the arithmetic of
the recognition method itself (no framing, DFT, convolution, attention, ...).

Two buffers need a formula to be drawn at all, because the method treats them
as stored inputs rather than computing them:

* the STFT window and the mel filterbank.  "GigaAM on MLX: the transcripts
  matched, but the model was broken", section "Trap 3", explains that the
  runtime must load the filterbank and window stored in the checkpoint instead
  of recomputing them.  Those buffers are not available here, so stand-ins are
  drawn with the textbook recipe named in "GigaAM v3 MLX", section "Frontend
  configuration" (HTK mel scale, no normalisation, 64 bins, 320-point FFT):
  a periodic Hann window and triangular HTK filters with f_min = 0 Hz and
  f_max = 8000 Hz (both limits are not printed on the pages; they are the
  plainest reading for 16 kHz audio).
* INT8 / INT6 / INT4 group-64 weights.  "GigaAM MLX port for Mac", section "How
  precision affects size and speed", says that each group of 64 weights shares
  one scale and measures 8, 6 and 4 bits.  Quantisation is an offline conversion
  step, so it lives with the inputs: the GPU path consumes (q, scale) and the
  oracle consumes q * scale.

Recipes (seeded with numpy PCG64):
  audio  C1-C4: sum of 3 sinusoids, f ~ U[200, 3000] Hz, amplitude 0.1 each,
         uniform random phase, plus N(0, 0.01) noise (0.01 is the standard
         deviation).
  audio  C5: linear chirp 100 -> 4000 Hz over the whole 300 s clip,
         amplitude 0.1, plus N(0, 0.02); cut into 15 x 20 s chunks.
  weights: matrices and biases N(0, 0.02); LayerNorm / BatchNorm gamma =
         1 + N(0, 0.02), beta ~ N(0, 0.02); BN running mean ~ N(0, 0.02),
         running var = 1 + |N(0, 0.02)|.  All rounded to fp16 (the checkpoints
         on the pages are fp16), window and filterbank stay fp32.
"""
from __future__ import annotations

import math
from typing import Dict, Tuple

import numpy as np

SAMPLE_RATE = 16000

# ---------------------------------------------------------------------------
# Model configurations
# ---------------------------------------------------------------------------

# Architecture shared by every configuration (frontend and subsampling).
_FRONT = dict(n_mels=64, n_fft=320, win=320, hop=160, sub_kernel=5,
              rope_base=5000.0, ln_eps=1e-5, bn_eps=1e-5)

V3 = dict(n_layers=16, d_model=768, n_heads=16, ffn_dim=3072, conv_kernel=31, **_FRONT)
LARGE = dict(n_layers=24, d_model=1024, n_heads=16, ffn_dim=4096, conv_kernel=31, **_FRONT)

PRECISIONS = {"fp32": 0, "fp16": 1, "int8_g64": 2, "int6_g64": 3, "int4_g64": 4}
QUANT_BITS = {"int8_g64": 8, "int6_g64": 6, "int4_g64": 4}

# The five benchmark / parity workloads.
WORKLOADS = {
    "c1_1s_b1_d768": dict(model=V3, n_classes=34, precision="fp16", kind="fixed",
                          batch=1, seconds=1.0, audio_seed=100),
    "c2_varlen_b32_d768": dict(model=V3, n_classes=34, precision="fp16", kind="uniform",
                               batch=32, min_seconds=2.0, max_seconds=20.0, audio_seed=101),
    "c3_20s_b64_d768": dict(model=V3, n_classes=257, precision="fp16", kind="fixed",
                            batch=64, seconds=20.0, audio_seed=102),
    "c4_30s_b32_d1024": dict(model=LARGE, n_classes=257, precision="fp16", kind="fixed",
                             batch=32, seconds=30.0, audio_seed=103),
    "c5_300s_chunks15_d1024_int8": dict(model=LARGE, n_classes=257, precision="int8_g64",
                                        kind="chirp", batch=15, seconds=20.0, audio_seed=104),
    # the same long-form input with 6- and 4-bit g64 weights ("GigaAM MLX port for
    # Mac", "How precision affects size and speed")
    "c5_300s_chunks15_d1024_int6": dict(model=LARGE, n_classes=257, precision="int6_g64",
                                        kind="chirp", batch=15, seconds=20.0, audio_seed=104),
    "c5_300s_chunks15_d1024_int4": dict(model=LARGE, n_classes=257, precision="int4_g64",
                                        kind="chirp", batch=15, seconds=20.0, audio_seed=104),
}


def model_config(model: dict, n_classes: int, precision: str, **overrides) -> dict:
    """Full configuration dict (same field names as the C ``gam_config``)."""
    cfg = dict(model)
    cfg.update(n_classes=int(n_classes), precision=precision)
    cfg.update(overrides)
    return cfg


def workload_config(name: str, **overrides) -> dict:
    w = WORKLOADS[name]
    return model_config(w["model"], w["n_classes"], w["precision"], **overrides)


# ---------------------------------------------------------------------------
# Audio
# ---------------------------------------------------------------------------

def _sinusoids(rng: np.random.Generator, n: int) -> np.ndarray:
    t = np.arange(n, dtype=np.float64) / SAMPLE_RATE
    x = np.zeros(n, dtype=np.float64)
    for _ in range(3):
        f = rng.uniform(200.0, 3000.0)
        ph = rng.uniform(0.0, 2.0 * math.pi)
        x += 0.1 * np.sin(2.0 * math.pi * f * t + ph)
    x += rng.normal(0.0, 0.01, size=n)
    return x.astype(np.float32)


def _chirp(rng: np.random.Generator, n: int) -> np.ndarray:
    t = np.arange(n, dtype=np.float64) / SAMPLE_RATE
    dur = n / SAMPLE_RATE
    f0, f1 = 100.0, 4000.0
    phase = 2.0 * math.pi * (f0 * t + (f1 - f0) * t * t / (2.0 * dur))
    x = 0.1 * np.sin(phase) + rng.normal(0.0, 0.02, size=n)
    return x.astype(np.float32)


def clip_lengths(name: str) -> np.ndarray:
    """Sample counts N_i of every clip of a workload (int64)."""
    w = WORKLOADS[name]
    if w["kind"] in ("fixed", "chirp"):
        return np.full(w["batch"], int(round(w["seconds"] * SAMPLE_RATE)), dtype=np.int64)
    rng = np.random.Generator(np.random.PCG64(w["audio_seed"] + 1000))
    lo = int(w["min_seconds"] * SAMPLE_RATE)
    hi = int(w["max_seconds"] * SAMPLE_RATE)
    u = rng.random(w["batch"])
    return (lo + np.floor(u * (hi - lo + 1))).astype(np.int64)


def workload_audio(name: str, clips: int | None = None) -> Tuple[np.ndarray, np.ndarray]:
    """Right-padded audio batch [B, Nmax] float32 and lengths [B] int32."""
    w = WORKLOADS[name]
    lens = clip_lengths(name)
    if clips is not None:
        lens = lens[:clips]
    rng = np.random.Generator(np.random.PCG64(w["audio_seed"]))
    B = len(lens)
    nmax = int(lens.max())
    audio = np.zeros((B, nmax), dtype=np.float32)
    if w["kind"] == "chirp":
        total = int(lens.sum())
        full = _chirp(rng, int(w["batch"] * w["seconds"] * SAMPLE_RATE))[:total]
        off = 0
        for i, n in enumerate(lens):
            audio[i, :n] = full[off:off + n]
            off += n
    else:
        for i, n in enumerate(lens):
            audio[i, :n] = _sinusoids(rng, int(n))
    return audio, lens.astype(np.int32)


def random_audio(lengths, seed: int) -> Tuple[np.ndarray, np.ndarray]:
    """Sinusoid+noise audio for arbitrary clip lengths (tests)."""
    lens = np.asarray(lengths, dtype=np.int64)
    rng = np.random.Generator(np.random.PCG64(seed))
    audio = np.zeros((len(lens), int(lens.max())), dtype=np.float32)
    for i, n in enumerate(lens):
        audio[i, :n] = _sinusoids(rng, int(n))
    return audio, lens.astype(np.int32)


# ---------------------------------------------------------------------------
# Frontend buffers (stand-ins for the checkpoint's stored window / filterbank)
# ---------------------------------------------------------------------------

def hann_window(win: int = 320) -> np.ndarray:
    """Periodic Hann window, fp32."""
    n = np.arange(win, dtype=np.float64)
    return (0.5 - 0.5 * np.cos(2.0 * math.pi * n / win)).astype(np.float32)


def htk_mel_filterbank(n_fft: int = 320, n_mels: int = 64, sample_rate: int = SAMPLE_RATE,
                       f_min: float = 0.0, f_max: float = 8000.0) -> np.ndarray:
    """Triangular HTK-scale filters, no normalisation: [n_fft//2+1, n_mels] fp32."""
    n_freqs = n_fft // 2 + 1
    bin_hz = np.linspace(0.0, sample_rate / 2.0, n_freqs)

    def to_mel(f):
        return 2595.0 * np.log10(1.0 + np.asarray(f, dtype=np.float64) / 700.0)

    def to_hz(m):
        return 700.0 * (10.0 ** (np.asarray(m, dtype=np.float64) / 2595.0) - 1.0)

    edges = to_hz(np.linspace(to_mel(f_min), to_mel(f_max), n_mels + 2))
    fb = np.zeros((n_freqs, n_mels), dtype=np.float64)
    for m in range(n_mels):
        lo, mid, hi = edges[m], edges[m + 1], edges[m + 2]
        rise = (bin_hz - lo) / (mid - lo)
        fall = (hi - bin_hz) / (hi - mid)
        fb[:, m] = np.maximum(0.0, np.minimum(rise, fall))
    return fb.astype(np.float32)


# ---------------------------------------------------------------------------
# Weights
# ---------------------------------------------------------------------------

def quantize_g64(w: np.ndarray, bits: int = 8) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric weight-only quantisation to `bits` (8, 6 or 4), groups of 64 along
    the input dim.

    w: [out, in] (or [out, in, 1]).  Returns q int8 of w's shape and scale fp16
    [out, in/64] with w ~= q * scale.  With qmax = 2^(bits-1) - 1: scale =
    fp16(max|w| / qmax) per group (1 when the group is all zero); q =
    clamp(round_half_even(w / scale), -qmax, qmax) computed in fp64 with the
    fp16-rounded scale.
    """
    if bits not in (8, 6, 4):
        raise ValueError("bits must be 8, 6 or 4")
    qmax = 2 ** (bits - 1) - 1
    shape = w.shape
    w2 = np.asarray(w, dtype=np.float64).reshape(shape[0], -1)
    out_f, in_f = w2.shape
    if in_f % 64:
        raise ValueError("input dimension must be a multiple of 64")
    g = w2.reshape(out_f, in_f // 64, 64)
    amax = np.abs(g).max(axis=2)
    scale = np.where(amax > 0, amax / qmax, 1.0).astype(np.float16)
    s64 = scale.astype(np.float64)[:, :, None]
    q = np.clip(np.rint(g / s64), -qmax, qmax).astype(np.int8)
    return q.reshape(shape), scale


def quantized_linear_names(cfg: dict):
    """Names of the linear weights stored quantised (g64) in the int*_g64 precisions."""
    names = []
    for l in range(cfg["n_layers"]):
        p = f"layers.{l}."
        for ffn in ("ffn1", "ffn2"):
            names += [p + ffn + ".linear1", p + ffn + ".linear2"]
        names += [p + "attn.linear_q", p + "attn.linear_k", p + "attn.linear_v", p + "attn.linear_out"]
        names += [p + "conv.pointwise1", p + "conv.pointwise2"]
    names.append("head")
    return names


def weight_shapes(cfg: dict) -> Dict[str, tuple]:
    """Every named tensor of the model, PyTorch layout (Linear [out,in], Conv1d [out,in,K])."""
    d, f, K = cfg["d_model"], cfg["ffn_dim"], cfg["conv_kernel"]
    nm, ks, C = cfg["n_mels"], cfg["sub_kernel"], cfg["n_classes"]
    s = {
        "frontend.window": (cfg["win"],),
        "frontend.mel_fb": (cfg["n_fft"] // 2 + 1, nm),
        "subsampling.conv1.weight": (d, nm, ks), "subsampling.conv1.bias": (d,),
        "subsampling.conv2.weight": (d, d, ks), "subsampling.conv2.bias": (d,),
    }
    for l in range(cfg["n_layers"]):
        p = f"layers.{l}."
        for ffn in ("ffn1", "ffn2"):
            s[p + ffn + ".norm.weight"] = (d,)
            s[p + ffn + ".norm.bias"] = (d,)
            s[p + ffn + ".linear1.weight"] = (f, d)
            s[p + ffn + ".linear1.bias"] = (f,)
            s[p + ffn + ".linear2.weight"] = (d, f)
            s[p + ffn + ".linear2.bias"] = (d,)
        s[p + "attn.norm.weight"] = (d,)
        s[p + "attn.norm.bias"] = (d,)
        for lin in ("linear_q", "linear_k", "linear_v", "linear_out"):
            s[p + "attn." + lin + ".weight"] = (d, d)
            s[p + "attn." + lin + ".bias"] = (d,)
        s[p + "conv.norm.weight"] = (d,)
        s[p + "conv.norm.bias"] = (d,)
        s[p + "conv.pointwise1.weight"] = (2 * d, d, 1)
        s[p + "conv.pointwise1.bias"] = (2 * d,)
        s[p + "conv.depthwise.weight"] = (d, 1, K)
        s[p + "conv.depthwise.bias"] = (d,)
        for bn in ("weight", "bias", "running_mean", "running_var"):
            s[p + "conv.bn." + bn] = (d,)
        s[p + "conv.pointwise2.weight"] = (d, d, 1)
        s[p + "conv.pointwise2.bias"] = (d,)
        s[p + "norm_out.weight"] = (d,)
        s[p + "norm_out.bias"] = (d,)
    s["head.weight"] = (C, d)
    s["head.bias"] = (C,)
    return s


def _is_gamma(name: str) -> bool:
    return name.endswith("norm.weight") or name.endswith("norm_out.weight") or name.endswith("bn.weight")


def random_weights(cfg: dict, seed: int = 0) -> Dict[str, np.ndarray]:
    """Seeded weights for ``cfg``.  fp16 tensors (fp32 window / filterbank).

    For the precisions "int8_g64", "int6_g64" and "int4_g64" each quantised
    linear ``X.weight`` is replaced by ``X.weight_q`` (int8 array holding q) and
    ``X.weight_scale`` (fp16 [out, in/64]).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out: Dict[str, np.ndarray] = {}
    for name, shape in weight_shapes(cfg).items():
        if name == "frontend.window":
            out[name] = hann_window(cfg["win"])
            continue
        if name == "frontend.mel_fb":
            out[name] = htk_mel_filterbank(cfg["n_fft"], cfg["n_mels"])
            continue
        if _is_gamma(name):
            v = 1.0 + rng.normal(0.0, 0.02, size=shape)
        elif name.endswith("running_var"):
            v = 1.0 + np.abs(rng.normal(0.0, 0.02, size=shape))
        else:
            v = rng.normal(0.0, 0.02, size=shape)
        out[name] = v.astype(np.float16)
    if cfg.get("precision") in QUANT_BITS:
        bits = QUANT_BITS[cfg["precision"]]
        for base in quantized_linear_names(cfg):
            w = out.pop(base + ".weight")
            q, s = quantize_g64(w, bits)
            out[base + ".weight_q"] = q
            out[base + ".weight_scale"] = s
    return out


# ---------------------------------------------------------------------------
# RNNT head (predictor LSTM + joint network)
# ---------------------------------------------------------------------------

RNNT = dict(pred_dim=320, joint_dim=320, max_symbols=10, joint_act="relu")


def rnnt_weight_shapes(d_model: int, n_classes: int, pred_dim: int = 320, joint_dim: int = 320) -> Dict[str, tuple]:
    """Named tensors of the RNNT head, PyTorch layout (embedding [C, P], LSTM
    weight_ih_l0 / weight_hh_l0 [4P, P] with two biases, Linear [out, in])."""
    P, J, C = pred_dim, joint_dim, n_classes
    return {"rnnt.embed.weight": (C, P),
            "rnnt.lstm.weight_ih_l0": (4 * P, P), "rnnt.lstm.weight_hh_l0": (4 * P, P),
            "rnnt.lstm.bias_ih_l0": (4 * P,), "rnnt.lstm.bias_hh_l0": (4 * P,),
            "rnnt.joint.enc.weight": (J, d_model), "rnnt.joint.enc.bias": (J,),
            "rnnt.joint.pred.weight": (J, P), "rnnt.joint.pred.bias": (J,),
            "rnnt.joint.out.weight": (C, J), "rnnt.joint.out.bias": (C,)}


def random_rnnt_weights(d_model: int, n_classes: int, seed: int = 7, pred_dim: int = 320, joint_dim: int = 320,
                        blank_bias: float = 7.0) -> Dict[str, np.ndarray]:
    """Seeded RNNT head weights, fp16.  Recipe: embedding N(0, 0.5); LSTM
    weights and both biases N(0, 0.05); joint enc / pred weights N(0, 0.05) and
    biases N(0, 0.02); joint out weights N(0, 0.1) and bias N(0, 0.1), plus
    `blank_bias` on the blank row (last class).  Random weights alone would
    rarely pick blank among 34 or 1025 classes, and the weak predictor path lets
    a frame that picks a symbol repeat it up to the per-frame cap; with the
    default offset, unit-variance encoder frames give about 0.7 (34 classes) to
    1.7 (1025 classes) symbols per frame on average, the order of a character
    or piece rate of speech at 40 ms frames."""
    rng = np.random.Generator(np.random.PCG64(seed))
    sd = {"rnnt.embed.weight": 0.5, "rnnt.lstm.weight_ih_l0": 0.05, "rnnt.lstm.weight_hh_l0": 0.05,
          "rnnt.lstm.bias_ih_l0": 0.05, "rnnt.lstm.bias_hh_l0": 0.05, "rnnt.joint.enc.weight": 0.05,
          "rnnt.joint.enc.bias": 0.02, "rnnt.joint.pred.weight": 0.05, "rnnt.joint.pred.bias": 0.02,
          "rnnt.joint.out.weight": 0.1, "rnnt.joint.out.bias": 0.1}
    out = {}
    for name, shape in rnnt_weight_shapes(d_model, n_classes, pred_dim, joint_dim).items():
        v = rng.normal(0.0, sd[name], size=shape)
        if name == "rnnt.joint.out.bias":
            v[-1] += blank_bias
        out[name] = v.astype(np.float16)
    return out

