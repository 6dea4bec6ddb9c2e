"""Pins of the oracle's rotary tables and rotary multi-head self-attention."""
import math

import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import synth
from conftest import read_golden


def test_rope_tables_vs_complex_recurrence():
    """cos/sin(t * w_i) obtained by repeated complex multiplication z_i^t,
    z_i = exp(1j * 5000^(-2i/dh)), instead of evaluating the angle."""
    g = read_golden("rope.txt")
    base = float(g["base"])
    dh = int(g["d_model"]) // int(g["n_heads"])
    assert dh == 48
    T = 40
    cos, sin = oracle.rope_tables(T, dh, base)
    half = dh // 2
    for i in range(half):
        z = complex(math.cos(base ** (-2.0 * i / dh)), math.sin(base ** (-2.0 * i / dh)))
        acc = 1.0 + 0.0j
        for t in range(T):
            assert cos[t, i] == pytest.approx(acc.real, abs=1e-12)
            assert sin[t, i] == pytest.approx(acc.imag, abs=1e-12)
            assert cos[t, i + half] == cos[t, i] and sin[t, i + half] == sin[t, i]
            acc *= z
    # position 0 is the identity rotation; channel pair 0 turns by exactly 1 rad per step
    assert np.all(cos[0] == 1.0) and np.all(sin[0] == 0.0)
    np.testing.assert_allclose(cos[:, 0], np.cos(np.arange(T)), atol=1e-15)


def test_rope_base_5000_vs_10000_gap():
    """The page reports that base-10000 tables 'diverged by almost 2'."""
    g = read_golden("rope.txt")
    dh = int(g["d_model"]) // int(g["n_heads"])
    for T, lo, hi in ((25, 0.5, 0.8), (100, float(g["table_gap_min"]), 2.0), (500, 1.99, 2.0)):
        c5, s5 = oracle.rope_tables(T, dh, float(g["base"]))
        c1, s1 = oracle.rope_tables(T, dh, float(g["wrong_base"]))
        gap = max(np.abs(c5 - c1).max(), np.abs(s5 - s1).max())
        assert lo < gap <= hi + 1e-12, (T, gap)


def test_apply_rope_is_complex_rotation():
    """With the halves convention each pair (x_i, x_{i+dh/2}) is the complex
    number x_i + 1j x_{i+dh/2} multiplied by exp(1j t w_i)."""
    rng = np.random.default_rng(0)
    T, H, dh = 7, 2, 8
    u = rng.normal(size=(T, H * dh))
    r = oracle.apply_rope(u, H, 5000.0)
    half = dh // 2
    w = 5000.0 ** (-2.0 * np.arange(half) / dh)
    for t in range(T):
        for h in range(H):
            x = u[t, h * dh:(h + 1) * dh]
            z = (x[:half] + 1j * x[half:]) * np.exp(1j * t * w)
            np.testing.assert_allclose(r[t, h * dh:h * dh + half], z.real, atol=1e-12)
            np.testing.assert_allclose(r[t, h * dh + half:(h + 1) * dh], z.imag, atol=1e-12)


def test_rope_relative_position_property():
    rng = np.random.default_rng(1)
    dh = 16
    a, b = rng.normal(size=(1, dh)), rng.normal(size=(1, dh))
    def rot(x, t):
        seq = np.zeros((t + 1, dh))
        seq[t] = x
        return oracle.apply_rope(seq, 1, 5000.0)[t]
    d1 = rot(a[0], 3) @ rot(b[0], 9)
    d2 = rot(a[0], 13) @ rot(b[0], 19)
    assert d1 == pytest.approx(d2, rel=1e-10)


def _attention_loops(q, k, v, n_valid):
    T, dh = q.shape
    out = np.zeros((T, v.shape[1]))
    for i in range(T):
        s = [sum(q[i, c] * k[j, c] for c in range(dh)) / math.sqrt(dh) for j in range(n_valid)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        for j in range(n_valid):
            out[i] += e[j] / z * v[j]
    return out


def test_masked_attention_vs_loops_and_garbage_keys():
    rng = np.random.default_rng(2)
    T, dh = 6, 5
    q, k, v = rng.normal(size=(3, T, dh))
    np.testing.assert_allclose(oracle.masked_attention(q, k, v), _attention_loops(q, k, v, T), rtol=1e-12)
    # append garbage keys/values and mask them: result must equal the clean one
    kg = np.concatenate([k, 1e3 * rng.normal(size=(4, dh))])
    vg = np.concatenate([v, 1e3 * rng.normal(size=(4, dh))])
    np.testing.assert_allclose(oracle.masked_attention(q, kg, vg, n_valid_keys=T),
                               oracle.masked_attention(q, k, v), rtol=1e-12)


def _mhsa_weights(d, rng, wq=None, wk=None, wv=None, wo=None):
    eye = np.eye(d)
    W = {}
    for name, m in (("linear_q", wq), ("linear_k", wk), ("linear_v", wv), ("linear_out", wo)):
        W[f"a.{name}.weight"] = rng.normal(size=(d, d)) if m is None else m
        W[f"a.{name}.bias"] = np.zeros(d)
    return W


def test_rotary_mhsa_uniform_attention_when_qk_zero():
    """Wq = Wk = 0: every score is 0, so each head averages V over the clip."""
    rng = np.random.default_rng(3)
    T, H, dh = 5, 2, 4
    d = H * dh
    cfg = dict(n_heads=H, rope_base=5000.0)
    u = rng.normal(size=(T, d))
    W = _mhsa_weights(d, rng, wq=np.zeros((d, d)), wk=np.zeros((d, d)), wv=np.eye(d), wo=np.eye(d))
    out = oracle.rotary_mhsa(u, W, "a", cfg, np.float64)
    np.testing.assert_allclose(out, np.tile(u.mean(axis=0), (T, 1)), rtol=1e-12)


def test_rotary_mhsa_rotates_input_before_projection():
    """Wq = Wk = Wv = Wo = I: scores are <R_s u_s, R_t u_t> per head, built
    here from explicit 2x2 rotation matrices; V is the unrotated input."""
    rng = np.random.default_rng(4)
    T, H, dh = 6, 2, 4
    d = H * dh
    base = 5000.0
    cfg = dict(n_heads=H, rope_base=base)
    u = rng.normal(size=(T, d))
    eye = np.eye(d)
    W = _mhsa_weights(d, rng, wq=eye, wk=eye, wv=eye, wo=eye)
    got = oracle.rotary_mhsa(u, W, "a", cfg, np.float64)
    half = dh // 2
    ref = np.zeros((T, d))
    for h in range(H):
        uh = u[:, h * dh:(h + 1) * dh]
        rot = np.zeros_like(uh)
        for t in range(T):
            for i in range(half):
                a = t * base ** (-2.0 * i / dh)
                R = np.array([[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]])
                rot[t, [i, i + half]] = R @ uh[t, [i, i + half]]
        ref[:, h * dh:(h + 1) * dh] = _attention_loops(rot, rot, uh, T)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
