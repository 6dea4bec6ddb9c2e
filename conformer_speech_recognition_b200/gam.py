"""Python binding of the C ABI in include/gam.h (ctypes, argument marshalling only).

Every function here has the name of the C entry point it calls.  Device
buffers are torch CUDA tensors (PyTorch provides memory and streams only);
lengths are host int32 arrays.  All compute runs in ``libgam.so``; there is no
fallback: if the library is missing this module raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgam.so")

GAM_FP32, GAM_FP16, GAM_INT8_G64, GAM_INT6_G64, GAM_INT4_G64 = 0, 1, 2, 3, 4
PRECISION = {"fp32": GAM_FP32, "fp16": GAM_FP16, "int8_g64": GAM_INT8_G64, "int6_g64": GAM_INT6_G64,
             "int4_g64": GAM_INT4_G64}
DTYPE_F32, DTYPE_F16, DTYPE_I8 = 0, 1, 2
(STAGE_SUBSAMPLING, STAGE_FFN1, STAGE_MHSA, STAGE_CONV, STAGE_FFN2, STAGE_LAYER) = range(6)

STATUS = {0: "GAM_OK", 1: "GAM_ERR_INVALID_ARG", 2: "GAM_ERR_SHAPE", 3: "GAM_ERR_CAPACITY", 4: "GAM_ERR_WEIGHTS",
          5: "GAM_ERR_UNSUPPORTED_DEVICE", 6: "GAM_ERR_CUDA", 7: "GAM_ERR_DEVICE_TIMEOUT"}

# Every entry point declared in include/gam.h.
EXPORTS = ("gam_status_string", "gam_last_error", "gam_plan_lengths", "gam_create", "gam_destroy", "gam_logmel",
           "gam_encode", "gam_encode_stage", "gam_ctc_greedy", "gam_ctc_greedy_frames", "gam_ctc_collapse",
           "gam_transcribe",
           "gam_device_status", "gam_profile_enable", "gam_profile_reset", "gam_profile_kinds",
           "gam_profile_kind_name", "gam_profile_read", "gam_graphs_enable", "gam_ctc_collapse_noalloc",
           "gam_rnnt_attach", "gam_rnnt_greedy", "gam_stream_create", "gam_stream_destroy", "gam_stream_reset",
           "gam_stream_push",
           "gam_debug_gemm", "gam_debug_wait_timeout", "gam_debug_inject_cuda_error")

GAM_NOALLOC_MAX_FRAMES = 1 << 20


class GamConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("ffn_dim", ctypes.c_int), ("conv_kernel", ctypes.c_int), ("n_mels", ctypes.c_int),
                ("n_fft", ctypes.c_int), ("win", ctypes.c_int), ("hop", ctypes.c_int),
                ("sub_kernel", ctypes.c_int), ("n_classes", ctypes.c_int), ("rope_base", ctypes.c_float),
                ("ln_eps", ctypes.c_float), ("bn_eps", ctypes.c_float), ("precision", ctypes.c_int),
                ("max_batch", ctypes.c_int), ("max_samples", ctypes.c_int64)]


class GamRnntConfig(ctypes.Structure):
    _fields_ = [("n_classes", ctypes.c_int), ("pred_dim", ctypes.c_int), ("joint_dim", ctypes.c_int),
                ("max_symbols", ctypes.c_int), ("joint_act", ctypes.c_int)]


class GamTensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("data", ctypes.c_void_p), ("dtype", ctypes.c_int),
                ("ndim", ctypes.c_int), ("shape", ctypes.c_int64 * 4)]


class GamError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.name = STATUS.get(status, str(status))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgam.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m conformer_speech_recognition_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32p, i64 = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_int64
        L.gam_status_string.restype = ctypes.c_char_p
        L.gam_status_string.argtypes = [ctypes.c_int]
        L.gam_last_error.restype = ctypes.c_char_p
        L.gam_last_error.argtypes = [vp]
        L.gam_plan_lengths.argtypes = [ctypes.POINTER(GamConfig), i32p, ctypes.c_int, i32p, i32p, i32p]
        L.gam_create.argtypes = [ctypes.POINTER(GamConfig), ctypes.POINTER(GamTensor), ctypes.c_int, ctypes.c_int,
                                 ctypes.POINTER(vp)]
        L.gam_destroy.argtypes = [vp]
        L.gam_logmel.argtypes = [vp, vp, i32p, ctypes.c_int, i64, vp, i32p, vp]
        L.gam_encode.argtypes = [vp, vp, i32p, ctypes.c_int, i64, vp, i32p, vp]
        L.gam_encode_stage.argtypes = [vp, vp, i32p, ctypes.c_int, i64, ctypes.c_int, ctypes.c_int, vp, vp]
        L.gam_ctc_greedy.argtypes = [vp, vp, i32p, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
        L.gam_ctc_greedy_frames.argtypes = [vp, vp, i32p, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
        L.gam_ctc_collapse.argtypes = [vp, vp, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        L.gam_transcribe.argtypes = [vp, vp, i32p, ctypes.c_int, i64, vp, vp, vp]
        L.gam_device_status.argtypes = [vp]
        L.gam_profile_enable.argtypes = [vp, ctypes.c_int]
        L.gam_profile_reset.argtypes = [vp]
        L.gam_profile_kinds.argtypes = []
        L.gam_profile_kind_name.restype = ctypes.c_char_p
        L.gam_profile_kind_name.argtypes = [ctypes.c_int]
        L.gam_profile_read.argtypes = [vp, ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
        L.gam_graphs_enable.argtypes = [vp, ctypes.c_int]
        L.gam_ctc_collapse_noalloc.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        L.gam_rnnt_attach.argtypes = [vp, ctypes.POINTER(GamRnntConfig), ctypes.POINTER(GamTensor), ctypes.c_int]
        L.gam_rnnt_greedy.argtypes = [vp, vp, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
        L.gam_stream_create.argtypes = [vp, ctypes.c_int64, ctypes.POINTER(vp)]
        L.gam_stream_destroy.argtypes = [vp]
        L.gam_stream_reset.argtypes = [vp]
        L.gam_stream_push.argtypes = [vp, vp, ctypes.c_int64, i32p, ctypes.c_int, i32p,
                                      ctypes.POINTER(ctypes.c_int64), vp]
        L.gam_debug_gemm.argtypes = [vp, ctypes.c_int, vp, ctypes.c_int, vp, vp, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, vp, ctypes.c_int, vp]
        L.gam_debug_wait_timeout.argtypes = [vp, ctypes.c_int64, ctypes.c_int]
        L.gam_debug_inject_cuda_error.argtypes = [vp, ctypes.c_int, ctypes.c_int]
        for name in EXPORTS:
            if name not in ("gam_status_string", "gam_last_error", "gam_profile_kind_name"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, ctx=None):
    if status != 0:
        msg = lib().gam_last_error(ctx.handle if ctx is not None else None)
        raise GamError(status, msg.decode() if msg else "")


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr_i32(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _dev_tensor(t, dtype, name: str, device=None):
    """Check that t is a contiguous CUDA tensor of `dtype` (on `device` if given):
    the C ABI reads it as a packed array through its data pointer."""
    import torch
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise GamError(1, f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise GamError(1, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise GamError(1, f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise GamError(1, f"{name} is on {t.device}, expected {device}")
    return t


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def make_config(cfg: dict, max_batch: int, max_samples: int) -> GamConfig:
    prec = cfg["precision"]
    return GamConfig(cfg["n_layers"], cfg["d_model"], cfg["n_heads"], cfg["ffn_dim"], cfg["conv_kernel"],
                     cfg["n_mels"], cfg["n_fft"], cfg["win"], cfg["hop"], cfg["sub_kernel"], cfg["n_classes"],
                     cfg["rope_base"], cfg["ln_eps"], cfg["bn_eps"],
                     PRECISION[prec] if isinstance(prec, str) else int(prec), int(max_batch), int(max_samples))


class Context:
    """Owns a gam_ctx handle (freed by gam_destroy / close())."""

    def __init__(self, handle, cfg: dict, max_batch: int, max_samples: int):
        self.handle = handle
        self.cfg = dict(cfg)
        self.max_batch = max_batch
        self.max_samples = max_samples
        self.config = make_config(cfg, max_batch, max_samples)

    def close(self):
        if self.handle:
            lib().gam_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gam_status_string(status: int) -> str:
    return lib().gam_status_string(status).decode()


def gam_plan_lengths(cfg: dict, lengths) -> Tuple[np.ndarray, np.ndarray, int, int]:
    """(frames F_i, valid encoder frames L'_i, F_max, T'_max) for sample counts."""
    ln = _i32(lengths)
    c = make_config(cfg, max(1, len(ln)), max(1280, int(ln.max()) if len(ln) else 1280))
    fr = np.zeros(len(ln), np.int32)
    el = np.zeros(len(ln), np.int32)
    dims = np.zeros(2, np.int32)
    _check(lib().gam_plan_lengths(ctypes.byref(c), _ptr_i32(ln), len(ln), _ptr_i32(fr), _ptr_i32(el), _ptr_i32(dims)))
    return fr, el, int(dims[0]), int(dims[1])


def _tensor_table(weights: Dict[str, np.ndarray]):
    keep = []
    arr = (GamTensor * len(weights))()
    for i, (name, w) in enumerate(weights.items()):
        w = np.ascontiguousarray(w)
        if w.dtype == np.float32:
            dt = DTYPE_F32
        elif w.dtype == np.float16:
            dt = DTYPE_F16
        elif w.dtype == np.int8:
            dt = DTYPE_I8
        else:
            w = np.ascontiguousarray(w.astype(np.float32))
            dt = DTYPE_F32
        nb = name.encode()
        keep += [w, nb]
        shape = (ctypes.c_int64 * 4)(*(list(w.shape) + [0] * (4 - w.ndim)))
        arr[i] = GamTensor(nb, w.ctypes.data, dt, w.ndim, shape)
    return arr, keep


def gam_create(cfg: dict, weights: Dict[str, np.ndarray], max_batch: int, max_samples: int,
               device: int = 0) -> Context:
    c = make_config(cfg, max_batch, max_samples)
    arr, keep = _tensor_table(weights)
    h = ctypes.c_void_p()
    st = lib().gam_create(ctypes.byref(c), arr, len(weights), device, ctypes.byref(h))
    if st != 0:
        raise GamError(st, lib().gam_last_error(None).decode())
    del keep
    return Context(h, cfg, max_batch, max_samples)


def gam_destroy(ctx: Context):
    ctx.close()


def gam_logmel(ctx: Context, audio, lengths, out=None, stream=None):
    import torch
    ln = _i32(lengths)
    _, _, fmax, _ = gam_plan_lengths(ctx.cfg, ln)
    _dev_tensor(audio, torch.float32, "audio")
    B, nmax = audio.shape
    if out is None:
        out = torch.empty((B, fmax, ctx.cfg["n_mels"]), dtype=torch.float32, device=audio.device)
    _dev_tensor(out, torch.float32, "out", audio.device)
    frames = np.zeros(B, np.int32)
    _check(lib().gam_logmel(ctx.handle, audio.data_ptr(), _ptr_i32(ln), B, nmax, out.data_ptr(), _ptr_i32(frames),
                            _stream(stream)), ctx)
    return out, frames


def gam_encode(ctx: Context, audio, lengths, out=None, stream=None):
    import torch
    ln = _i32(lengths)
    _, _, _, tmax = gam_plan_lengths(ctx.cfg, ln)
    _dev_tensor(audio, torch.float32, "audio")
    B, nmax = audio.shape
    if out is None:
        out = torch.empty((B, tmax, ctx.cfg["d_model"]), dtype=torch.float32, device=audio.device)
    _dev_tensor(out, torch.float32, "out", audio.device)
    enc_len = np.zeros(B, np.int32)
    _check(lib().gam_encode(ctx.handle, audio.data_ptr(), _ptr_i32(ln), B, nmax, out.data_ptr(), _ptr_i32(enc_len),
                            _stream(stream)), ctx)
    return out, enc_len


def gam_encode_stage(ctx: Context, audio, lengths, layer: int, stage: int, out=None, stream=None):
    import torch
    ln = _i32(lengths)
    _, _, _, tmax = gam_plan_lengths(ctx.cfg, ln)
    _dev_tensor(audio, torch.float32, "audio")
    B, nmax = audio.shape
    if out is None:
        out = torch.empty((B, tmax, ctx.cfg["d_model"]), dtype=torch.float32, device=audio.device)
    _dev_tensor(out, torch.float32, "out", audio.device)
    _check(lib().gam_encode_stage(ctx.handle, audio.data_ptr(), _ptr_i32(ln), B, nmax, layer, stage, out.data_ptr(),
                                  _stream(stream)), ctx)
    return out


def gam_ctc_greedy(ctx: Context, enc, enc_len, want_logp: bool = False, stream=None, tokens=None, counts=None,
                   logp=None):
    """Greedy CTC decoding of enc [B, T, d]; tokens / counts / logp may be passed in
    (preallocated CUDA tensors, so repeated calls keep their pointers)."""
    import torch
    el = _i32(enc_len)
    _dev_tensor(enc, torch.float32, "enc")
    B, tmax, _ = enc.shape
    C = ctx.cfg["n_classes"]
    if tokens is None:
        tokens = torch.empty((B, tmax), dtype=torch.int32, device=enc.device)
    if counts is None:
        counts = torch.empty((B,), dtype=torch.int32, device=enc.device)
    if logp is None and want_logp:
        logp = torch.empty((B, tmax, C), dtype=torch.float32, device=enc.device)
    _dev_tensor(tokens, torch.int32, "tokens", enc.device)
    _dev_tensor(counts, torch.int32, "counts", enc.device)
    if logp is not None:
        _dev_tensor(logp, torch.float32, "logp", enc.device)
    _check(lib().gam_ctc_greedy(ctx.handle, enc.data_ptr(), _ptr_i32(el), B, tmax,
                                logp.data_ptr() if logp is not None else None, tokens.data_ptr(), counts.data_ptr(),
                                _stream(stream)), ctx)
    return tokens, counts, logp


def gam_ctc_greedy_frames(ctx: Context, enc, enc_len, stream=None, tokens=None, frames=None, counts=None):
    """Greedy CTC decoding with the first frame of each token: (tokens, frames,
    counts) as CUDA int32 tensors [B, T], [B, T], [B]."""
    import torch
    el = _i32(enc_len)
    _dev_tensor(enc, torch.float32, "enc")
    B, tmax, _ = enc.shape
    if tokens is None:
        tokens = torch.empty((B, tmax), dtype=torch.int32, device=enc.device)
    if frames is None:
        frames = torch.empty((B, tmax), dtype=torch.int32, device=enc.device)
    if counts is None:
        counts = torch.empty((B,), dtype=torch.int32, device=enc.device)
    for t, n in ((tokens, "tokens"), (frames, "frames"), (counts, "counts")):
        _dev_tensor(t, torch.int32, n, enc.device)
    _check(lib().gam_ctc_greedy_frames(ctx.handle, enc.data_ptr(), _ptr_i32(el), B, tmax, tokens.data_ptr(),
                                       frames.data_ptr(), counts.data_ptr(), _stream(stream)), ctx)
    return tokens, frames, counts


def gam_ctc_collapse(ctx: Context, logits, lengths, stream=None):
    import torch
    ln = _i32(lengths)
    _dev_tensor(logits, torch.float32, "logits")
    B, tmax, C = logits.shape
    tokens = torch.empty((B, tmax), dtype=torch.int32, device=logits.device)
    counts = torch.empty((B,), dtype=torch.int32, device=logits.device)
    _check(lib().gam_ctc_collapse(ctx.handle, logits.data_ptr(), _ptr_i32(ln), B, tmax, C, tokens.data_ptr(),
                                  counts.data_ptr(), _stream(stream)), ctx)
    return tokens, counts


def gam_transcribe(ctx: Context, audio_host, lengths, tokens_host=None, counts_host=None, stream=None):
    """audio_host: host float32 [B, Nmax] (numpy or pinned torch CPU tensor)."""
    ln = _i32(lengths)
    _, _, _, tmax = gam_plan_lengths(ctx.cfg, ln)
    B, nmax = audio_host.shape
    if tokens_host is None:
        tokens_host = np.zeros((B, tmax), np.int32)
    if counts_host is None:
        counts_host = np.zeros(B, np.int32)

    def addr(a):
        return a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data

    _check(lib().gam_transcribe(ctx.handle, addr(audio_host), _ptr_i32(ln), B, nmax, addr(tokens_host),
                                addr(counts_host), _stream(stream)), ctx)
    return tokens_host, counts_host


def gam_device_status(ctx: Context):
    _check(lib().gam_device_status(ctx.handle), ctx)


def gam_profile_enable(ctx: Context, mask=True):
    """mask: True / -1 = every kernel family, False / 0 = none, else a bit mask of families."""
    if mask is True:
        mask = -1
    elif mask is False:
        mask = 0
    _check(lib().gam_profile_enable(ctx.handle, int(mask)), ctx)


def gam_profile_reset(ctx: Context):
    _check(lib().gam_profile_reset(ctx.handle), ctx)


def gam_profile_kinds() -> int:
    return lib().gam_profile_kinds()


def gam_profile_kind_name(kind: int) -> str:
    return lib().gam_profile_kind_name(kind).decode()


def gam_profile_read(ctx: Context, kind: int) -> Tuple[float, int]:
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    _check(lib().gam_profile_read(ctx.handle, kind, ctypes.byref(ms), ctypes.byref(n)), ctx)
    return ms.value, n.value


def gam_profile_all(ctx: Context) -> Dict[str, Tuple[float, int]]:
    return {gam_profile_kind_name(k): gam_profile_read(ctx, k) for k in range(gam_profile_kinds())}


def gam_ctc_collapse_noalloc(logits, lengths_dev, tokens, counts, stream=None):
    """Greedy decoding with no context and no allocation inside the call.

    logits: CUDA f32 [B, T, C]; lengths_dev: CUDA int32 [B]; tokens (CUDA int32
    [B, T]) and counts (CUDA int32 [B]) are written.  The caller allocates all
    four; the library keeps its per-frame scratch in a fixed device array."""
    import torch
    _dev_tensor(logits, torch.float32, "logits")
    for t, dt, n in ((lengths_dev, torch.int32, "lengths_dev"), (tokens, torch.int32, "tokens"),
                     (counts, torch.int32, "counts")):
        _dev_tensor(t, dt, n, logits.device)
    B, T, C = logits.shape
    if tuple(lengths_dev.shape) != (B,) or tuple(tokens.shape) != (B, T) or tuple(counts.shape) != (B,):
        raise GamError(1, "lengths_dev [B], tokens [B, T] and counts [B] must match logits [B, T, C]")
    _check(lib().gam_ctc_collapse_noalloc(logits.data_ptr(), lengths_dev.data_ptr(), B, T, C, tokens.data_ptr(),
                                          counts.data_ptr(), _stream(stream)))
    return tokens, counts


def gam_rnnt_attach(ctx: Context, rnnt_cfg: dict, weights: Dict[str, np.ndarray]):
    """Attach the RNNT head: rnnt_cfg has n_classes, pred_dim, joint_dim,
    max_symbols and joint_act ("relu" or "tanh"); weights named as in gam.h."""
    act = rnnt_cfg.get("joint_act", "relu")
    c = GamRnntConfig(int(rnnt_cfg["n_classes"]), int(rnnt_cfg.get("pred_dim", 320)),
                      int(rnnt_cfg.get("joint_dim", 320)), int(rnnt_cfg.get("max_symbols", 10)),
                      0 if act in ("relu", 0) else 1)
    arr, keep = _tensor_table(weights)
    _check(lib().gam_rnnt_attach(ctx.handle, ctypes.byref(c), arr, len(weights)), ctx)
    del keep
    ctx.rnnt_cfg = dict(rnnt_cfg)


def gam_rnnt_greedy(ctx: Context, enc, enc_len, max_tokens: Optional[int] = None, stream=None, tokens=None,
                    frames=None, counts=None):
    """Greedy RNNT decoding of enc [B, T, d]: (tokens [B, max_tokens], frames
    [B, max_tokens], counts [B]) as CUDA int32 tensors."""
    import torch
    el = _i32(enc_len)
    _dev_tensor(enc, torch.float32, "enc")
    B, tmax, _ = enc.shape
    if max_tokens is None:
        max_tokens = tmax * int(ctx.rnnt_cfg.get("max_symbols", 10))
    if tokens is None:
        tokens = torch.empty((B, max_tokens), dtype=torch.int32, device=enc.device)
    if frames is None:
        frames = torch.empty((B, max_tokens), dtype=torch.int32, device=enc.device)
    if counts is None:
        counts = torch.empty((B,), dtype=torch.int32, device=enc.device)
    for t, n in ((tokens, "tokens"), (frames, "frames"), (counts, "counts")):
        _dev_tensor(t, torch.int32, n, enc.device)
    _check(lib().gam_rnnt_greedy(ctx.handle, enc.data_ptr(), _ptr_i32(el), B, tmax, int(max_tokens),
                                 tokens.data_ptr(), frames.data_ptr(), counts.data_ptr(), _stream(stream)), ctx)
    return tokens, frames, counts


class Stream:
    """Pseudo-streaming recogniser over a context (gam_stream_*)."""

    def __init__(self, ctx: Context, window_samples: int = 30 * 16000):
        h = ctypes.c_void_p()
        _check(lib().gam_stream_create(ctx.handle, int(window_samples), ctypes.byref(h)), ctx)
        self.handle, self.ctx, self.window = h, ctx, int(window_samples)
        _, _, _, self.t_cap = gam_plan_lengths(ctx.cfg, [max(1280, self.window)])
        self._tok = np.zeros(self.t_cap, np.int32)

    def push(self, samples, stream=None):
        """Append host float32 samples; returns (tokens of the current window, index
        of the window's first sample in the stream)."""
        x = np.ascontiguousarray(np.asarray(samples, dtype=np.float32))
        cnt = np.zeros(1, np.int32)
        start = ctypes.c_int64()
        _check(lib().gam_stream_push(self.handle, x.ctypes.data if x.size else None, x.size, _ptr_i32(self._tok),
                                     self.t_cap, _ptr_i32(cnt), ctypes.byref(start), _stream(stream)), self.ctx)
        return self._tok[:min(int(cnt[0]), self.t_cap)].copy(), int(start.value)

    def reset(self):
        _check(lib().gam_stream_reset(self.handle), self.ctx)

    def close(self):
        if self.handle:
            lib().gam_stream_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gam_stream_create(ctx: Context, window_samples: int = 30 * 16000) -> Stream:
    return Stream(ctx, window_samples)


def gam_graphs_enable(ctx: Context, on: bool = True):
    """Replay CUDA graphs for repeated identical calls (on by default)."""
    _check(lib().gam_graphs_enable(ctx.handle, 1 if on else 0), ctx)


def gam_debug_gemm(ctx: Context, impl: int, a, w, bias, out, stream=None):
    """out += a . w^T + bias (a, w fp16 CUDA tensors; bias, out fp32)."""
    M, K = a.shape
    N = w.shape[0]
    _check(lib().gam_debug_gemm(ctx.handle, impl, a.data_ptr(), a.stride(0), w.data_ptr(), bias.data_ptr(), M, N, K,
                                out.data_ptr(), out.stride(0), _stream(stream)), ctx)
    return out


def gam_debug_wait_timeout(ctx: Context, limit_ns: int, skip_k_block: int = -1):
    """The next tensor-core GEMM's waits give up after limit_ns; with
    skip_k_block >= 0 its producer leaves that k-block's stage empty."""
    _check(lib().gam_debug_wait_timeout(ctx.handle, int(limit_ns), int(skip_k_block)), ctx)


def gam_debug_inject_cuda_error(ctx: Context, cuda_error: int, count: int = 1):
    _check(lib().gam_debug_inject_cuda_error(ctx.handle, cuda_error, count), ctx)
