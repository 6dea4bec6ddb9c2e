"""Pins of the oracle's CTC head, greedy collapse and INT8 g64 dequantisation."""
import itertools

import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import synth
from conftest import read_golden_rows


def test_collapse_hand_cases():
    rows = read_golden_rows("collapse.txt")
    assert len(rows) >= 6
    for blank, seq, expected in rows:
        seq = [int(t) for t in seq.split()]
        exp = [int(t) for t in expected.split()]
        assert oracle.greedy_collapse(seq, int(blank)) == exp


def test_collapse_vs_groupby_bruteforce():
    rng = np.random.default_rng(0)
    for _ in range(500):
        blank = int(rng.integers(1, 5))
        seq = rng.integers(0, blank + 1, size=int(rng.integers(0, 20))).tolist()
        ref = [k for k, _ in itertools.groupby(seq) if k != blank]
        assert oracle.greedy_collapse(seq, blank) == ref


def test_collapse_frames_hand_cases():
    """Each kept symbol carries the first frame of its run."""
    assert oracle.greedy_collapse_frames([5, 5, 7, 7], 33) == ([5, 7], [0, 2])
    assert oracle.greedy_collapse_frames([33, 5, 33, 5, 5], 33) == ([5, 5], [1, 3])
    assert oracle.greedy_collapse_frames([33, 33], 33) == ([], [])
    rng = np.random.default_rng(3)
    for _ in range(200):
        blank = int(rng.integers(1, 4))
        seq = rng.integers(0, blank + 1, size=int(rng.integers(0, 15))).tolist()
        sym, fr = oracle.greedy_collapse_frames(seq, blank)
        assert sym == oracle.greedy_collapse(seq, blank)
        assert all(seq[f] == k and (f == 0 or seq[f - 1] != k) for k, f in zip(sym, fr))
        assert fr == sorted(fr) and len(set(fr)) == len(fr)


def test_ctc_head_logsoftmax_and_first_argmax():
    rng = np.random.default_rng(1)
    d, C, T = 6, 5, 4
    W = {"head.weight": rng.normal(size=(C, d)), "head.bias": np.zeros(C)}
    enc = rng.normal(size=(T, d))
    z, logp, a = oracle.ctc_head(enc, W)
    np.testing.assert_allclose(np.exp(logp).sum(axis=1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(z - logp, np.broadcast_to(np.log(np.exp(z).sum(axis=1))[:, None], z.shape), rtol=1e-12)
    np.testing.assert_array_equal(a, [int(np.argmax(r)) for r in z])
    # ties: lowest index wins
    W2 = {"head.weight": np.zeros((C, d)), "head.bias": np.array([0.0, 2.0, 2.0, 1.0, 2.0])}
    _, _, a2 = oracle.ctc_head(enc, W2)
    assert np.all(a2 == 1)


def test_int8_g64_round_trip_bound():
    rng = np.random.default_rng(2)
    w = (rng.normal(0, 0.02, size=(16, 256))).astype(np.float16)
    w[3, 64:128] = 0  # an all-zero group
    q, s = synth.quantize_g64(w)
    assert q.dtype == np.int8 and s.dtype == np.float16 and s.shape == (16, 4)
    assert np.abs(q).max() <= 127
    back = oracle.dequant_g64(q, s)
    err = np.abs(back - w.astype(np.float64))
    bound = np.repeat(s.astype(np.float64), 64, axis=1) / 2
    assert np.all(err <= bound * (1 + 1e-9) + 1e-12)
    assert s[3, 1] == 1.0 and np.all(q[3, 64:128] == 0)
    # the largest magnitude of each group maps to +-127 (up to fp16 rounding of the scale)
    g = np.abs(q.reshape(16, 4, 64)).max(axis=2)
    assert np.all((g >= 126) | (s == 1.0))


@pytest.mark.parametrize("bits,qmax", [(8, 127), (6, 31), (4, 7)])
def test_g64_round_trip_bound_every_width(bits, qmax):
    """q * s reproduces w within s / 2 per element at 8, 6 and 4 bits; each
    group's largest magnitude maps to +-qmax; hand case: a group of 64 values
    -7 .. 7 (times 0.01) at 4 bits has scale 0.01 in fp16 and q = the integers."""
    rng = np.random.default_rng(bits)
    w = rng.normal(0, 0.02, size=(8, 192)).astype(np.float16)
    w[2, :64] = 0
    q, s = synth.quantize_g64(w, bits)
    assert q.dtype == np.int8 and np.abs(q).max() <= qmax
    back = oracle.dequant_g64(q, s)
    bound = np.repeat(s.astype(np.float64), 64, axis=1) / 2
    assert np.all(np.abs(back - w.astype(np.float64)) <= bound * (1 + 1e-9) + 1e-12)
    g = np.abs(q.reshape(8, 3, 64)).max(axis=2)
    assert np.all((g >= qmax - 1) | (s == 1.0))
    assert s[2, 0] == 1.0 and np.all(q[2, :64] == 0)
    if bits == 4:
        ints = np.tile(np.arange(-7, 8), 5)[:64].astype(np.float64)
        q4, s4 = synth.quantize_g64((ints * 0.01)[None, :], 4)
        assert s4[0, 0] == np.float16(0.01)
        assert np.array_equal(q4[0], ints.astype(np.int8))


def test_int8_weights_replace_every_linear():
    cfg = synth.model_config(dict(synth.LARGE, n_layers=1, d_model=128, n_heads=2, ffn_dim=256), 257, "int8_g64")
    W = synth.random_weights(cfg)
    names = synth.quantized_linear_names(cfg)
    assert len(names) == 11
    for n in names:
        assert n + ".weight" not in W and W[n + ".weight_q"].dtype == np.int8
        w, b = oracle.get_linear(W, n)
        assert w.shape[0] == b.shape[0]
