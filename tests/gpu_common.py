"""Shared helpers of the GPU parity tests: cached seeded weights, contexts and
oracle results, and the comparison metrics with the tolerances the tests use."""
import functools

import numpy as np

import oracle
from conformer_speech_recognition_b200 import gam, synth

# fp32 build mode: max |delta| per layer output (and per stage).
TOL_FP32_LAYER = 1e-4
# fp32 frontend: max |delta| of the log-mel features.  The DFT runs in fp32 with
# blocked summation (10 partial sums of 32 samples): first-order error of a DFT
# coefficient <= (32 + 10) u sum|x w cos|, u = 2^-24, so the relative error of a
# power bin is <= 2 * 42 u * rho with rho = sum|x w cos| / |X| (<= ~40 for the
# synthetic tones + noise floor): 2 * 42 * 6e-8 * 40 = 2.0e-4 on the log scale.
# (The pages' own frontend ports report 3e-5 and 4.2e-4 against PyTorch fp32.)
TOL_LOGMEL = 2e-4


def logmel_bound_tensor_core(x, window, fb, win=320, hop=160):
    """Per-element bound on |log-mel error| of the tensor-core frontend (3xTF32
    DFT with fp32 accumulation), derived from its arithmetic on the clip x:

      DFT:   each product term x w cos is formed from tf32 parts as
             hi*hi + lo*hi + hi*lo; the tf32 roundings of the lo parts and the
             dropped lo*lo leave <= 3 * 2^-22 of |x w cos|.  The accumulator
             takes 120 steps (3 products x 40 instructions of 8 samples), each
             allowed 2^-22 of the running sum's bound (one rounding of the
             8-product group and one of the add), so
             |dRe_k| <= eps * S^c_k,  eps = 3 * 2^-22 + 120 * 2^-22,
             S^c_k = sum_n |x_n w_n cos(2 pi k n / 320)|  (sin likewise).
      power: |dP_k| <= 2 |Re| dRe + dRe^2 + 2 |Im| dIm + dIm^2 + 2^-22 P_k.
      mel:   |dmel| <= sum_k fb[k, m] |dP_k| + 2^-24 * (rows in the sum) * mel.
      log:   |dlog| <= dmel / (mel - dmel) + 2^-22 |log mel|.
    Returns the bound [F, n_mels] and the exact log-mel in fp64."""
    import numpy as np
    x = np.asarray(x, np.float64)
    F = 1 + (len(x) - win) // hop
    idx = np.arange(F)[:, None] * hop + np.arange(win)[None, :]
    fr = x[idx] * np.asarray(window, np.float64)[None, :]
    k = np.arange(win // 2 + 1)[:, None]
    n = np.arange(win)[None, :]
    ang = 2 * np.pi * ((k * n) % win) / win
    c, s = np.cos(ang), np.sin(ang)
    re, im = fr @ c.T, fr @ s.T
    sc, ss = np.abs(fr) @ np.abs(c).T, np.abs(fr) @ np.abs(s).T
    eps = 3 * 2.0 ** -22 + 120 * 2.0 ** -22
    dre, dim_ = eps * sc, eps * ss
    P = re ** 2 + im ** 2
    dP = 2 * np.abs(re) * dre + dre ** 2 + 2 * np.abs(im) * dim_ + dim_ ** 2 + 2.0 ** -22 * P
    fb = np.asarray(fb, np.float64)
    mel = P @ fb
    rows = (fb != 0).sum(axis=0)[None, :]
    dmel = dP @ fb + 2.0 ** -24 * rows * mel
    mel_c = np.clip(mel, 1e-9, 1e9)
    lo = np.maximum(mel - dmel, 1e-9)
    bound = np.where(mel - dmel > 1e-9, dmel / lo, np.log(np.maximum(mel + dmel, 1e-9) / 1e-9))
    return bound + 2.0 ** -22 * np.abs(np.log(mel_c)), np.log(mel_c)


# fp16 / INT8 product modes: relative Frobenius error, max |delta|, argmax agreement.
TOL_REL_FRO = 1e-2
TOL_MAX_ABS = 5e-2
MIN_ARGMAX_AGREE = 0.995


def small_model(d=256, heads=4, ffn=512, layers=2, K=31):
    return dict(synth.V3, n_layers=layers, d_model=d, n_heads=heads, ffn_dim=ffn, conv_kernel=K)


@functools.lru_cache(maxsize=8)
def _weights(model_items, n_classes, precision, seed):
    cfg = synth.model_config(dict(model_items), n_classes, precision)
    return synth.random_weights(cfg, seed=seed)


def config_and_weights(model: dict, n_classes: int, precision: str, seed: int = 0):
    """(config, seeded weights) -- weights cached per (model, classes, precision, seed)."""
    cfg = synth.model_config(dict(model), n_classes, precision)
    return cfg, _weights(tuple(sorted(model.items())), n_classes, precision, seed)


def oracle_clip(audio_row, n, W, cfg, dump=False, n_layers=None):
    d = {} if dump else None
    enc = oracle.encode_clip(audio_row[:n].astype(np.float64), W, cfg, np.float64, dump=d, n_layers=n_layers)
    return enc, d


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def max_abs(a, b):
    return float(np.abs(a - b).max()) if a.size else 0.0


def to_torch(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()
