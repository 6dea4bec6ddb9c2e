"""Pins of the oracle's Conv1d subsampling and length bookkeeping."""
import numpy as np

import oracle
from conformer_speech_recognition_b200 import synth
from conftest import read_golden


def _conv1d_loops(x, w, b, stride, pad):
    T, cin = x.shape
    cout, _, K = w.shape
    Tout = (T + 2 * pad - K) // stride + 1
    y = np.zeros((Tout, cout))
    for t in range(Tout):
        for o in range(cout):
            acc = b[o]
            for k in range(K):
                src = stride * t + k - pad
                if 0 <= src < T:
                    for c in range(cin):
                        acc += w[o, c, k] * x[src, c]
            y[t, o] = acc
    return y


def test_conv1d_vs_loops():
    rng = np.random.default_rng(0)
    for T in (1, 2, 5, 9, 10):
        x = rng.normal(size=(T, 3))
        w = rng.normal(size=(4, 3, 5))
        b = rng.normal(size=4)
        np.testing.assert_allclose(oracle.conv1d(x, w, b, 2, 2), _conv1d_loops(x, w, b, 2, 2), rtol=1e-12, atol=1e-12)


def test_conv1d_is_cross_correlation():
    # a single tap at k = pad + 1 reads the NEXT input row (no kernel flip)
    x = np.arange(8, dtype=np.float64)[:, None]
    w = np.zeros((1, 1, 5))
    w[0, 0, 3] = 1.0
    y = oracle.conv1d(x, w, None, 1, 2)[:, 0]
    np.testing.assert_array_equal(y, np.r_[np.arange(1, 8), 0.0])


def test_lengths_match_printed_shapes():
    g = read_golden("shapes.txt")
    for s, f, t in zip(g["samples"], g["frames"], g["enc_frames"]):
        plan = oracle.clip_lengths_plan(int(s), synth.V3)
        assert plan["F"] == int(f)
        assert plan["T2"] == int(t)
    p = oracle.clip_lengths_plan(16000, synth.V3)
    assert (p["T1"], p["T2"], p["L1"], p["L2"]) == (50, 25, 49, 24)
    p = oracle.clip_lengths_plan(320000, synth.V3)
    assert (p["T1"], p["T2"], p["L1"], p["L2"]) == (1000, 500, 999, 499)
    # shortest clip with one valid encoder frame: L1 >= 3 needs F >= 7 frames -> 1280 samples
    assert oracle.clip_lengths_plan(1280, synth.V3)["L2"] == 1
    assert oracle.clip_lengths_plan(1279, synth.V3)["L2"] == 0


def test_valid_rows_do_not_see_padding():
    """Reading R3: valid outputs are unchanged when garbage rows follow the clip."""
    rng = np.random.default_rng(5)
    cfg = synth.model_config(dict(synth.V3, d_model=8), 34, "fp16")
    W = {"subsampling.conv1.weight": rng.normal(size=(8, 64, 5)),
         "subsampling.conv1.bias": rng.normal(size=8),
         "subsampling.conv2.weight": rng.normal(size=(8, 8, 5)),
         "subsampling.conv2.bias": rng.normal(size=8)}
    for F in (5, 6, 7, 8, 23, 24):
        mel = rng.normal(size=(F, 64))
        ref = oracle.subsample(mel, W, cfg)
        assert ref.shape[0] == oracle.valid_len_after_stride2(oracle.valid_len_after_stride2(F))
        padded = np.concatenate([mel, 100.0 * rng.normal(size=(6, 64))])
        h = np.maximum(oracle.conv1d(padded, W["subsampling.conv1.weight"], W["subsampling.conv1.bias"], 2, 2), 0)
        y = np.maximum(oracle.conv1d(h, W["subsampling.conv2.weight"], W["subsampling.conv2.bias"], 2, 2), 0)
        np.testing.assert_allclose(y[:ref.shape[0]], ref, rtol=1e-12, atol=1e-12)
