"""Pins of the oracle's frontend (framing, DFT power, mel filterbank, log).

Each check ties the oracle to something other than itself: shapes printed on
the pages, a brute-force O(N^2) DFT written with explicit loops, Parseval's
identity, closed-form spectra of a constant and of a pure bin cosine, and the
HTK mel scale's anchor values.
"""
import math

import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import synth
from conftest import read_golden

CFG = synth.model_config(synth.V3, 34, "fp16")


def test_frontend_constants_match_pages():
    g = read_golden("frontend.txt")
    assert int(g["sample_rate"]) == synth.SAMPLE_RATE
    assert int(g["n_mels"]) == CFG["n_mels"]
    assert int(g["n_fft"]) == CFG["n_fft"]
    assert int(g["win"]) == CFG["win"]
    assert int(g["hop"]) == CFG["hop"]
    assert float(g["log_clip_min"]) == oracle.gigaam.LOG_CLIP_MIN
    assert float(g["log_clip_max"]) == oracle.gigaam.LOG_CLIP_MAX


def test_frame_counts_match_printed_shapes():
    g = read_golden("shapes.txt")
    for s, f in zip(g["samples"], g["frames"]):
        assert oracle.n_frames(int(s), 320, 160) == int(f)
    # degenerate: shorter than one window -> no frame; exactly one window -> 1
    assert oracle.n_frames(319) == 0
    assert oracle.n_frames(320) == 1
    assert oracle.n_frames(479) == 1
    assert oracle.n_frames(480) == 2


def _dft_power_bruteforce(frame, window, n_fft):
    """|sum_n x[n] w[n] e^{-2 pi i k n / N}|^2 by explicit loops."""
    out = []
    for k in range(n_fft // 2 + 1):
        re = 0.0
        im = 0.0
        for n in range(n_fft):
            a = 2.0 * math.pi * k * n / n_fft
            re += frame[n] * window[n] * math.cos(a)
            im -= frame[n] * window[n] * math.sin(a)
        out.append(re * re + im * im)
    return np.array(out)


def test_power_spectrum_vs_bruteforce_dft():
    rng = np.random.default_rng(1)
    n_fft = 320
    window = synth.hann_window(n_fft).astype(np.float64)
    frames = rng.normal(size=(2, n_fft))
    P = oracle.power_spectrum(frames, window, n_fft)
    for i in range(2):
        ref = _dft_power_bruteforce(frames[i], window, n_fft)
        np.testing.assert_allclose(P[i], ref, rtol=1e-10, atol=1e-9)


def test_power_spectrum_parseval():
    rng = np.random.default_rng(2)
    n_fft = 320
    window = synth.hann_window(n_fft).astype(np.float64)
    frames = rng.normal(size=(4, n_fft))
    P = oracle.power_spectrum(frames, window, n_fft)
    energy = ((frames * window) ** 2).sum(axis=1)
    # one-sided spectrum: DC and Nyquist once, all others twice
    two_sided = P[:, 0] + P[:, -1] + 2.0 * P[:, 1:-1].sum(axis=1)
    np.testing.assert_allclose(two_sided / n_fft, energy, rtol=1e-12)


def test_power_spectrum_special_cases():
    n = 320
    ones = np.ones(n)
    # constant frame, rectangular window: all energy in bin 0, |X0| = n * c
    c = 0.25
    P = oracle.power_spectrum(np.full((1, n), c), ones, n)[0]
    assert P[0] == pytest.approx((n * c) ** 2, rel=1e-12)
    assert np.all(P[1:] < 1e-18)
    # pure cosine at bin 7: |X7| = n/2, zero elsewhere
    t = np.arange(n)
    P = oracle.power_spectrum(np.cos(2 * math.pi * 7 * t / n)[None, :], ones, n)[0]
    assert P[7] == pytest.approx((n / 2) ** 2, rel=1e-12)
    assert np.delete(P, 7).max() < 1e-16
    # periodic Hann on a constant: X0 = c * n/2, X1 = -c * n/4, rest 0
    w = synth.hann_window(n).astype(np.float64)
    P = oracle.power_spectrum(np.full((1, n), 1.0), w, n)[0]
    assert P[0] == pytest.approx((n / 2) ** 2, rel=1e-6)
    assert P[1] == pytest.approx((n / 4) ** 2, rel=1e-6)
    assert P[2:].max() < 1e-6


def test_htk_mel_filterbank_against_definition():
    fb = synth.htk_mel_filterbank(320, 64).astype(np.float64)
    assert fb.shape == (161, 64)
    # HTK mel anchors: 2595*log10(1 + f/700); 700 Hz -> 2595*log10(2); 1000 Hz ~ 1000 mel
    mel = lambda f: 2595.0 * math.log10(1.0 + f / 700.0)
    assert mel(700.0) == pytest.approx(2595.0 * math.log10(2.0))
    assert abs(mel(1000.0) - 1000.0) < 0.05
    # filter m is a unit-peak triangle between edges m and m+2 (equally spaced in mel),
    # evaluated at the bin centres k * 50 Hz: compare with piecewise-linear interpolation
    mmax = mel(8000.0)
    edges_mel = np.linspace(0.0, mmax, 66)
    edges_hz = 700.0 * (10 ** (edges_mel / 2595.0) - 1.0)
    bins = np.arange(161) * 50.0
    for m in range(64):
        ref = np.interp(bins, edges_hz[m:m + 3], [0.0, 1.0, 0.0], left=0.0, right=0.0)
        np.testing.assert_allclose(fb[:, m], ref, atol=1e-6)
    assert fb.max() <= 1.0 + 1e-6
    assert np.all(fb >= 0)
    # no normalisation: every filter keeps a peak near 1 only if a bin falls near its centre;
    # the high filters (wide triangles) sum to more than 1 (unnormalised area)
    assert fb[:, -1].sum() > 1.0


def test_log_mel_clip_and_shape():
    cfg = CFG
    w = synth.hann_window(320)
    fb = synth.htk_mel_filterbank(320, 64)
    # silence -> every bin clipped to 1e-9
    z = oracle.log_mel(np.zeros(16000), w, fb, cfg)
    g = read_golden("shapes.txt")
    assert z.shape == (int(g["frames"][0]), 64)
    np.testing.assert_allclose(z, math.log(1e-9))
    # huge values clip at 1e9
    big = oracle.log_mel(np.full(320, 1e6), w, fb, cfg)
    assert big.max() == pytest.approx(math.log(1e9))


def test_log_mel_vs_bruteforce_small_clip():
    cfg = CFG
    w = synth.hann_window(320).astype(np.float64)
    fb = synth.htk_mel_filterbank(320, 64).astype(np.float64)
    audio, _ = synth.random_audio([640], seed=3)
    x = audio[0].astype(np.float64)
    got = oracle.log_mel(x, w, fb, cfg)
    assert got.shape == (3, 64)
    for f in range(3):
        frame = x[f * 160: f * 160 + 320]
        P = _dft_power_bruteforce(frame, w, 320)
        ref = np.log(np.clip(P @ fb, 1e-9, 1e9))
        np.testing.assert_allclose(got[f], ref, rtol=1e-9, atol=1e-9)
