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
