"""Plain NumPy definition of the GigaAM encoder + CTC path (oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Nothing here is tuned:
every step follows the pages' description in their order, on one clip at a time
and on its valid frames only.  ``dtype`` selects fp64 (checking) or fp32 (the
timed CPU baseline).

Sources (page title, section):
  [MLX-trap]  "GigaAM on MLX: the transcripts matched, but the model was broken":
              "What we're porting", "Trap 1: the RoPE base is 5000, not 10000",
              "Trap 2: RoPE before the projections", "Trap 3: mel filters",
              "Trap 4: weight layout and precision".
  [RNNT-card] "GigaAM v3 RNNT -- MLX (Apple Silicon)": "Notes for other runtimes".
  [Port-Mac]  "GigaAM MLX port for Mac": "What is inside the model",
              "How precision affects size and speed", "Where the time goes".
  [v3-MLX]    "GigaAM v3 MLX": "Frontend configuration", "Architecture details",
              "Validation".
  [Port-ru]   Russian original of [Port-Mac]: the pipeline list under
              "What is inside the model" (audio -> log-mel -> 2 conv layers ->
              Conformer blocks FFN/attention/convolution/FFN -> CTC -> decoding).

Readings where the pages are silent (each also listed in the design notes):
  R1 depthwise kernel size is a config field (31 in the benchmark configs).
  R2 every linear / conv layer has a bias.
  R3 valid length after each stride-2 conv is floor((L - 1) / 2).
  R4 rotate_half uses the halves convention, positions start at 0.
  R5 attention scale 1/sqrt(d_head), output projection with bias.
  R6 LayerNorm and BatchNorm eps 1e-5; each block ends with a LayerNorm.
  R7 macaron FFNs are added with weight 1/2.
  R10 rows at or beyond the valid length are zero for the depthwise conv.
  R11 argmax takes the lowest index among equal maxima; collapse merges
      repeats first, then drops blanks.
  R12 INT8 g64 weights are used as q * scale.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "n_frames", "conv_tensor_len", "valid_len_after_stride2", "clip_lengths_plan",
    "frame_signal", "power_spectrum", "log_mel",
    "conv1d", "subsample",
    "layer_norm", "swish", "glu", "batch_norm_eval", "depthwise_conv1d",
    "rope_tables", "rotate_half", "apply_rope", "masked_attention",
    "feed_forward", "rotary_mhsa", "conv_module", "conformer_layer",
    "dequant_g64", "get_linear",
    "encode_clip", "ctc_head", "greedy_collapse", "greedy_collapse_frames", "transcribe_clip",
    "oracle_weight_inventory",
]

LOG_CLIP_MIN = 1e-9
LOG_CLIP_MAX = 1e9


# ---------------------------------------------------------------------------
# Lengths
# ---------------------------------------------------------------------------

def n_frames(n_samples: int, win: int = 320, hop: int = 160) -> int:
    """Frame count of center=false framing ([v3-MLX] "Frontend configuration":
    window 320, hop 160, center false).  A frame starts every ``hop`` samples
    and must fit whole inside the clip."""
    if n_samples < win:
        return 0
    return 1 + (n_samples - win) // hop


def conv_tensor_len(t: int, k: int = 5, s: int = 2, p: int = 2) -> int:
    """Output length of a zero-padded Conv1d (tensor length, padded frames
    included).  [MLX-trap] "What we're porting": two stride-2 Conv1d layers."""
    return (t + 2 * p - k) // s + 1


def valid_len_after_stride2(length: int) -> int:
    """Reading R3: valid frames after one stride-2, kernel-5, pad-2 conv.

    With L = floor((T - 1) / 2) the last valid output t = L - 1 reads input rows
    up to 2t + 2 = 2L <= T - 1, so every valid output sees valid input only."""
    return max((length - 1) // 2, 0)


def clip_lengths_plan(n_samples: int, cfg: dict) -> dict:
    """All lengths of one clip: frames F, tensor lengths T1/T', valid L1/L'."""
    F = n_frames(n_samples, cfg["win"], cfg["hop"])
    k = cfg["sub_kernel"]
    p = k // 2
    T1 = conv_tensor_len(F, k, 2, p)
    T2 = conv_tensor_len(T1, k, 2, p)
    L1 = valid_len_after_stride2(F)
    L2 = valid_len_after_stride2(L1)
    return dict(F=F, T1=T1, T2=T2, L1=L1, L2=L2)


# ---------------------------------------------------------------------------
# Frontend  ([v3-MLX] "Frontend configuration"; [RNNT-card] "Notes for other
# runtimes": stored window and filterbank, center=False, log(clip(x,1e-9,1e9)))
# ---------------------------------------------------------------------------

def frame_signal(x: np.ndarray, win: int, hop: int) -> np.ndarray:
    """[F, win] matrix of frames, frame f = x[f*hop : f*hop + win]."""
    F = n_frames(len(x), win, hop)
    idx = np.arange(F)[:, None] * hop + np.arange(win)[None, :]
    return x[idx]


def power_spectrum(frames: np.ndarray, window: np.ndarray, n_fft: int) -> np.ndarray:
    """|rfft(frame * window)|^2 (power 2.0), [F, n_fft//2 + 1]."""
    X = np.fft.rfft(frames * window[None, :], n=n_fft, axis=1)
    return X.real ** 2 + X.imag ** 2


def log_mel(x: np.ndarray, window: np.ndarray, mel_fb: np.ndarray, cfg: dict,
            dtype=np.float64) -> np.ndarray:
    """Log-mel features of one clip, time-major [F, n_mels].

    The pages print features as [n_mels, F] ([v3-MLX] "Validation": [64, 99]);
    this oracle keeps time on the first axis.  The filterbank is applied as a
    plain matrix product with the stored buffer ([MLX-trap] "Trap 3")."""
    x = np.asarray(x, dtype=dtype)
    fr = frame_signal(x, cfg["win"], cfg["hop"])
    P = power_spectrum(fr, np.asarray(window, dtype=dtype), cfg["n_fft"])
    mel = P @ np.asarray(mel_fb, dtype=dtype)
    return np.log(np.clip(mel, LOG_CLIP_MIN, LOG_CLIP_MAX)).astype(dtype)


# ---------------------------------------------------------------------------
# Conv1d subsampling ([MLX-trap] "What we're porting": two Conv1d layers with
# stride 2; [v3-MLX] "Architecture details": Conv1D subsampling, factor 4)
# ---------------------------------------------------------------------------

def conv1d(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray], stride: int, pad: int) -> np.ndarray:
    """Cross-correlation Conv1d on time-major input (PyTorch semantics).

    x: [T, C_in]; w: [C_out, C_in, K] (PyTorch layout, [MLX-trap] "Trap 4");
    y[t, o] = b[o] + sum_k sum_c w[o, c, k] * x[stride*t + k - pad, c],
    with x = 0 outside [0, T)."""
    T, cin = x.shape
    cout, cin_w, K = w.shape
    assert cin == cin_w
    Tout = (T + 2 * pad - K) // stride + 1
    xp = np.zeros((T + 2 * pad, cin), dtype=x.dtype)
    xp[pad:pad + T] = x
    y = np.zeros((Tout, cout), dtype=x.dtype)
    if b is not None:
        y += b[None, :]
    for k in range(K):
        rows = xp[k: k + stride * (Tout - 1) + 1: stride]
        y += rows @ w[:, :, k].T
    return y


def subsample(mel: np.ndarray, W: Dict[str, np.ndarray], cfg: dict, dtype=np.float64) -> np.ndarray:
    """conv1 + ReLU, conv2 + ReLU over the full clip, then keep the valid rows
    L' (reading R3).  Returns [L', d]."""
    k = cfg["sub_kernel"]
    p = k // 2
    w1 = W["subsampling.conv1.weight"].astype(dtype)
    b1 = W["subsampling.conv1.bias"].astype(dtype)
    w2 = W["subsampling.conv2.weight"].astype(dtype)
    b2 = W["subsampling.conv2.bias"].astype(dtype)
    h = np.maximum(conv1d(mel.astype(dtype), w1, b1, 2, p), 0)
    y = np.maximum(conv1d(h, w2, b2, 2, p), 0)
    L1 = valid_len_after_stride2(mel.shape[0])
    L2 = valid_len_after_stride2(L1)
    return y[:L2]


# ---------------------------------------------------------------------------
# Elementwise / normalisation pieces (textbook Conformer; [RNNT-card] "Notes
# for other runtimes": only RoPE placement and base differ from the textbook)
# ---------------------------------------------------------------------------

def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def swish(x: np.ndarray) -> np.ndarray:
    """SiLU / Swish, x * sigmoid(x) ([Port-Mac] "Where the time goes": SiLU)."""
    return x / (1.0 + np.exp(-x))


def glu(h: np.ndarray) -> np.ndarray:
    """GLU over the channel axis: first half times sigmoid(second half)."""
    d = h.shape[-1] // 2
    return h[..., :d] / (1.0 + np.exp(-h[..., d:]))


def batch_norm_eval(x: np.ndarray, gamma, beta, mean, var, eps: float) -> np.ndarray:
    """Inference BatchNorm with running statistics, unfolded."""
    return (x - mean) / np.sqrt(var + eps) * gamma + beta


def depthwise_conv1d(x: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Per-channel Conv1d over time, 'same' zero padding (K-1)/2.

    x: [T, d] (rows beyond the clip are zero, reading R10); w: [d, 1, K]."""
    T, d = x.shape
    K = w.shape[-1]
    pad = (K - 1) // 2
    xp = np.zeros((T + 2 * pad, d), dtype=x.dtype)
    xp[pad:pad + T] = x
    y = np.zeros_like(x) + b[None, :]
    for k in range(K):
        y += xp[k:k + T] * w[:, 0, k][None, :]
    return y


# ---------------------------------------------------------------------------
# Rotary attention ([MLX-trap] "Trap 1" (base = pos_emb_max_len = 5000) and
# "Trap 2" (rotate the raw, head-split input before linear_q / linear_k; the
# same rotated input feeds Q and K; V is not rotated))
# ---------------------------------------------------------------------------

def rope_tables(T: int, d_head: int, base: float = 5000.0, dtype=np.float64):
    """cos/sin tables [T, d_head]: angle(t, i) = t * base^(-2i/d_head) for the
    first half, repeated for the second half (halves convention, R4)."""
    half = d_head // 2
    inv_freq = base ** (-(2.0 * np.arange(half, dtype=np.float64)) / d_head)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv_freq[None, :]
    ang = np.concatenate([ang, ang], axis=1)
    return np.cos(ang).astype(dtype), np.sin(ang).astype(dtype)


def rotate_half(x: np.ndarray) -> np.ndarray:
    """[x1, x2] -> [-x2, x1] on the last axis."""
    h = x.shape[-1] // 2
    return np.concatenate([-x[..., h:], x[..., :h]], axis=-1)


def apply_rope(u: np.ndarray, n_heads: int, base: float) -> np.ndarray:
    """x * cos + rotate_half(x) * sin per head on u: [T, d] (offset 0)."""
    T, d = u.shape
    dh = d // n_heads
    cos, sin = rope_tables(T, dh, base, u.dtype)
    uh = u.reshape(T, n_heads, dh)
    r = uh * cos[:, None, :] + rotate_half(uh) * sin[:, None, :]
    return r.reshape(T, d)


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_valid_keys: Optional[int] = None):
    """softmax(q k^T / sqrt(d_head) + mask) v for one head; q,k,v [T, d_head].
    Keys at index >= n_valid_keys are masked out (key-padding mask)."""
    dh = q.shape[-1]
    s = (q @ k.T) / math.sqrt(dh)
    if n_valid_keys is not None:
        s = s.copy()
        s[:, n_valid_keys:] = -np.inf
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ v


def dequant_g64(q: np.ndarray, scale: np.ndarray, dtype=np.float64) -> np.ndarray:
    """w = q * scale, one fp16 scale per group of 64 input weights (R12;
    [Port-Mac] "How precision affects size and speed")."""
    shape = q.shape
    q2 = q.reshape(shape[0], -1).astype(dtype)
    s = np.repeat(scale.astype(dtype), 64, axis=1)
    return (q2 * s).reshape(shape)


def get_linear(W: Dict[str, np.ndarray], name: str, dtype=np.float64):
    """(weight [out, in], bias [out]) of a linear / pointwise layer in dtype."""
    if name + ".weight" in W:
        w = W[name + ".weight"].astype(dtype)
    else:
        w = dequant_g64(W[name + ".weight_q"], W[name + ".weight_scale"], dtype)
    w = w.reshape(w.shape[0], -1)
    return w, W[name + ".bias"].astype(dtype)


def feed_forward(u: np.ndarray, W, prefix: str, dtype) -> np.ndarray:
    """Linear -> SiLU -> Linear ([Port-Mac] "Where the time goes")."""
    w1, b1 = get_linear(W, prefix + ".linear1", dtype)
    w2, b2 = get_linear(W, prefix + ".linear2", dtype)
    return swish(u @ w1.T + b1) @ w2.T + b2


def rotary_mhsa(u: np.ndarray, W, prefix: str, cfg: dict, dtype) -> np.ndarray:
    """Multi-head self-attention with RoPE on the raw (normalised) input.

    u is what the attention module receives (after its pre-LayerNorm).  Per
    [MLX-trap] "Trap 2": u_rot = RoPE(u split into heads); Q = linear_q(u_rot),
    K = linear_k(u_rot), V = linear_v(u); output = linear_out(concat heads)."""
    T, d = u.shape
    H = cfg["n_heads"]
    dh = d // H
    wq, bq = get_linear(W, prefix + ".linear_q", dtype)
    wk, bk = get_linear(W, prefix + ".linear_k", dtype)
    wv, bv = get_linear(W, prefix + ".linear_v", dtype)
    wo, bo = get_linear(W, prefix + ".linear_out", dtype)
    u_rot = apply_rope(u, H, cfg["rope_base"])
    q = (u_rot @ wq.T + bq).reshape(T, H, dh)
    k = (u_rot @ wk.T + bk).reshape(T, H, dh)
    v = (u @ wv.T + bv).reshape(T, H, dh)
    o = np.empty((T, H, dh), dtype=u.dtype)
    for h in range(H):
        o[:, h, :] = masked_attention(q[:, h], k[:, h], v[:, h])
    return o.reshape(T, d) @ wo.T + bo


def conv_module(u: np.ndarray, W, prefix: str, cfg: dict, dtype) -> np.ndarray:
    """Pointwise -> GLU -> depthwise -> BatchNorm -> Swish -> pointwise
    (textbook Conformer convolution module; [Port-ru] pipeline list)."""
    w1, b1 = get_linear(W, prefix + ".pointwise1", dtype)
    w2, b2 = get_linear(W, prefix + ".pointwise2", dtype)
    g = glu(u @ w1.T + b1)
    y = depthwise_conv1d(g, W[prefix + ".depthwise.weight"].astype(dtype),
                         W[prefix + ".depthwise.bias"].astype(dtype))
    y = batch_norm_eval(y, W[prefix + ".bn.weight"].astype(dtype), W[prefix + ".bn.bias"].astype(dtype),
                        W[prefix + ".bn.running_mean"].astype(dtype),
                        W[prefix + ".bn.running_var"].astype(dtype), cfg["bn_eps"])
    return swish(y) @ w2.T + b2


def _ln(x, W, name, cfg, dtype):
    return layer_norm(x, W[name + ".weight"].astype(dtype), W[name + ".bias"].astype(dtype), cfg["ln_eps"])


def conformer_layer(x: np.ndarray, W, l: int, cfg: dict, dtype=np.float64,
                    taps: Optional[list] = None) -> np.ndarray:
    """One block: FFN(1/2) -> rotary MHSA -> conv module -> FFN(1/2) -> LayerNorm
    ([Port-ru] "24 blocks: FFN, attention, convolution, FFN"; R6, R7)."""
    p = f"layers.{l}."
    x = x + 0.5 * feed_forward(_ln(x, W, p + "ffn1.norm", cfg, dtype), W, p + "ffn1", dtype)
    if taps is not None:
        taps.append(x.copy())
    x = x + rotary_mhsa(_ln(x, W, p + "attn.norm", cfg, dtype), W, p + "attn", cfg, dtype)
    if taps is not None:
        taps.append(x.copy())
    x = x + conv_module(_ln(x, W, p + "conv.norm", cfg, dtype), W, p + "conv", cfg, dtype)
    if taps is not None:
        taps.append(x.copy())
    x = x + 0.5 * feed_forward(_ln(x, W, p + "ffn2.norm", cfg, dtype), W, p + "ffn2", dtype)
    if taps is not None:
        taps.append(x.copy())
    x = _ln(x, W, p + "norm_out", cfg, dtype)
    if taps is not None:
        taps.append(x.copy())
    return x


def encode_clip(audio: np.ndarray, W, cfg: dict, dtype=np.float64, dump: Optional[dict] = None,
                n_layers: Optional[int] = None) -> np.ndarray:
    """Encoder output [L', d] of one clip (valid frames only).

    ``dump`` (a dict) receives every stage: "mel" [F, n_mels], "x0" [L', d] and
    "layers" = list over layers of the 5 stage outputs (after FFN1, MHSA, conv,
    FFN2, final LayerNorm), the layer-by-layer localisation method of
    [MLX-trap] "Trap 1"."""
    mel = log_mel(audio, W["frontend.window"], W["frontend.mel_fb"], cfg, dtype)
    x = subsample(mel, W, cfg, dtype)
    if dump is not None:
        dump["mel"] = mel
        dump["x0"] = x.copy()
        dump["layers"] = []
    nl = cfg["n_layers"] if n_layers is None else n_layers
    for l in range(nl):
        taps = [] if dump is not None else None
        x = conformer_layer(x, W, l, cfg, dtype, taps)
        if dump is not None:
            dump["layers"].append(taps)
    return x


# ---------------------------------------------------------------------------
# CTC head and greedy decoding ([Port-ru] pipeline: "CTC layer: probability of
# each symbol at each step"; "decoding: repeats and blank symbols are removed";
# [RNNT-card] "Notes for other runtimes": blank = len(vocabulary))
# ---------------------------------------------------------------------------

def ctc_head(enc: np.ndarray, W, dtype=np.float64):
    """logits, log-probabilities [T, C] and first-index argmax [T] (R11)."""
    w, b = get_linear(W, "head", dtype)
    z = enc.astype(dtype) @ w.T + b
    m = z.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(z - m).sum(axis=1, keepdims=True))
    return z, z - lse, np.argmax(z, axis=1).astype(np.int32)


def greedy_collapse(a, blank: int) -> List[int]:
    """Merge runs of equal symbols, then drop blanks (R11)."""
    out: List[int] = []
    prev = None
    for s in a:
        s = int(s)
        if s != prev and s != blank:
            out.append(s)
        prev = s
    return out


def greedy_collapse_frames(a, blank: int):
    """greedy_collapse with the frame where each kept symbol's run starts:
    (symbols, frames).  The frame places a symbol in time, which is what joins
    the transcripts of overlapping long-form chunks ([v3-MLX] "Long-form
    transcription": 20 s chunks with 0-2 s of overlap)."""
    out: List[int] = []
    frames: List[int] = []
    prev = None
    for t, s in enumerate(a):
        s = int(s)
        if s != prev and s != blank:
            out.append(s)
            frames.append(t)
        prev = s
    return out, frames


def transcribe_clip(audio: np.ndarray, W, cfg: dict, dtype=np.float64) -> dict:
    enc = encode_clip(audio, W, cfg, dtype)
    z, logp, a = ctc_head(enc, W, dtype)
    return dict(enc=enc, logits=z, logp=logp, argmax=a,
                tokens=greedy_collapse(a, cfg["n_classes"] - 1))


# ---------------------------------------------------------------------------
# Inventory of tensors the oracle reads (pinned against the pages' totals)
# ---------------------------------------------------------------------------

def oracle_weight_inventory(cfg: dict) -> Dict[str, tuple]:
    """Shape of every parameter tensor this oracle reads, by name (fp16 mode).
    BatchNorm running statistics are buffers, listed separately by the caller
    via the ``running_`` prefix."""
    d, f, K, C = cfg["d_model"], cfg["ffn_dim"], cfg["conv_kernel"], cfg["n_classes"]
    inv = {"subsampling.conv1.weight": (d, cfg["n_mels"], cfg["sub_kernel"]),
           "subsampling.conv1.bias": (d,),
           "subsampling.conv2.weight": (d, d, cfg["sub_kernel"]),
           "subsampling.conv2.bias": (d,)}
    for l in range(cfg["n_layers"]):
        p = f"layers.{l}."
        for n in ("ffn1", "ffn2"):
            inv.update({p + n + ".norm.weight": (d,), p + n + ".norm.bias": (d,),
                        p + n + ".linear1.weight": (f, d), p + n + ".linear1.bias": (f,),
                        p + n + ".linear2.weight": (d, f), p + n + ".linear2.bias": (d,)})
        inv.update({p + "attn.norm.weight": (d,), p + "attn.norm.bias": (d,)})
        for n in ("linear_q", "linear_k", "linear_v", "linear_out"):
            inv.update({p + "attn." + n + ".weight": (d, d), p + "attn." + n + ".bias": (d,)})
        inv.update({p + "conv.norm.weight": (d,), p + "conv.norm.bias": (d,),
                    p + "conv.pointwise1.weight": (2 * d, d, 1), p + "conv.pointwise1.bias": (2 * d,),
                    p + "conv.depthwise.weight": (d, 1, K), p + "conv.depthwise.bias": (d,),
                    p + "conv.bn.weight": (d,), p + "conv.bn.bias": (d,),
                    p + "conv.bn.running_mean": (d,), p + "conv.bn.running_var": (d,),
                    p + "conv.pointwise2.weight": (d, d, 1), p + "conv.pointwise2.bias": (d,),
                    p + "norm_out.weight": (d,), p + "norm_out.bias": (d,)})
    inv.update({"head.weight": (C, d), "head.bias": (C,)})
    return inv
