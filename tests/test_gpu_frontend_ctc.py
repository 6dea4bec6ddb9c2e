"""GPU parity of the log-mel frontend and of the CTC decoder, through the C ABI."""
import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import gam, synth
from gpu_common import TOL_LOGMEL, config_and_weights, logmel_bound_tensor_core, max_abs, small_model, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def small_ctx():
    cfg, W = config_and_weights(small_model(), 34, "fp32")
    ctx = gam.gam_create(cfg, W, 8, 200000)
    yield cfg, W, ctx
    ctx.close()


def test_logmel_parity_ragged(small_ctx):
    cfg, W, ctx = small_ctx
    lengths = [16000, 1280, 16159, 4321, 48000, 160001]
    audio, lens = synth.random_audio(lengths, seed=7)
    mel, frames = gam.gam_logmel(ctx, to_torch(audio), lens)
    mel = mel.cpu().numpy()
    for i, n in enumerate(lens):
        ref = oracle.log_mel(audio[i, :n].astype(np.float64), W["frontend.window"], W["frontend.mel_fb"], cfg)
        assert frames[i] == ref.shape[0]
        assert max_abs(mel[i, :frames[i]], ref) <= TOL_LOGMEL, i
        assert np.all(mel[i, frames[i]:] == 0)


@pytest.mark.parametrize("precision", ["fp16", "int8_g64"])
def test_logmel_product_context_parity(precision):
    """fp16 / INT8 contexts: gam_logmel runs the tensor-core frontend that
    gam_encode uses (3xTF32 DFT, power, filterbank and log in one kernel).  Its
    log-mel must match the oracle element by element within the bound derived
    from that arithmetic (logmel_bound_tensor_core), and overall within 4.23e-4,
    the largest log-mel difference the pages report between their port and the
    fp32 reference ("GigaAM v3 MLX", "Validation"), on
    a ragged batch with a quiet clip (tones at 1e-4, noise 1e-5), a loud one
    (tones at 0.9) and clips of 1280 samples and of a ragged number of frames,
    with the padded frames zero."""
    cfg, W = config_and_weights(small_model(layers=1), 34, precision)
    lengths = [16000, 1280, 37123, 48000, 4321, 160001]
    audio, lens = synth.random_audio(lengths, seed=19)
    audio[0] *= 1e-3   # quiet: tones at 1e-4, noise sigma 1e-5
    audio[3] *= 9.0    # loud: tones at 0.9
    ctx = gam.gam_create(cfg, W, len(lens), int(max(lens)))
    mel, frames = gam.gam_logmel(ctx, to_torch(audio), lens)
    mel = mel.cpu().numpy()
    worst = 0.0
    tightest = np.inf
    for i, n in enumerate(lens):
        x = audio[i, :n].astype(np.float64)
        ref = oracle.log_mel(x, W["frontend.window"], W["frontend.mel_fb"], cfg)
        bound, exact = logmel_bound_tensor_core(x, W["frontend.window"], W["frontend.mel_fb"])
        assert np.abs(exact - ref).max() < 1e-9  # the bound is about the same quantity the oracle computes
        assert frames[i] == ref.shape[0]
        err = np.abs(mel[i, :frames[i]] - ref)
        worst = max(worst, float(err.max()))
        assert np.all(err <= bound), (i, float((err / bound).max()))
        tightest = min(tightest, float((bound - err).min()))
        assert err.max() <= 4.23e-4, (i, float(err.max()))
        assert np.all(mel[i, frames[i]:] == 0)
    print(precision, "worst log-mel max|delta|", worst, "smallest bound slack", tightest)
    ctx.close()


def test_logmel_shape_printed_on_pages(small_ctx):
    cfg, W, ctx = small_ctx
    audio, lens = synth.random_audio([16000], seed=8)
    mel, frames = gam.gam_logmel(ctx, to_torch(audio), lens)
    assert tuple(mel.shape) == (1, 99, 64) and frames[0] == 99


def _crafted_logits(rng, B, T, C):
    z = rng.normal(size=(B, T, C)).astype(np.float32)
    blank = C - 1
    # runs of the same winner, blank runs and exact ties between two classes
    for b in range(B):
        for t in range(0, T, 7):
            z[b, t:t + 3, 5 % C] += 10.0
        for t in range(3, T, 11):
            z[b, t, blank] += 20.0
        for t in range(2, T, 13):
            m = z[b, t].max() + 1.0
            z[b, t, 1] = m
            z[b, t, 4] = m  # tie: lowest index (1) must win
        z[b, 9::23, :] = -np.inf  # all -inf: numpy's argmax gives index 0
        z[b, 10::29, 3] = np.nan  # a NaN ranks above every number, the first NaN wins
        z[b, 10::29, 6] = np.nan
    return z


@pytest.mark.parametrize("C", [34, 257, 1025])
def test_ctc_collapse_bit_exact(small_ctx, C):
    cfg, W, ctx = small_ctx
    rng = np.random.default_rng(C)
    B, T = 6, 300
    z = _crafted_logits(rng, B, T, C)
    lens = np.array([300, 0, 1, 299, 150, 17], np.int32)
    tok, cnt = gam.gam_ctc_collapse(ctx, to_torch(z), lens)
    tok, cnt = tok.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        a = np.argmax(z[b, :lens[b]], axis=1)
        ref = oracle.greedy_collapse(a, C - 1)
        assert cnt[b] == len(ref)
        assert tok[b, :cnt[b]].tolist() == ref
        assert np.all(tok[b, cnt[b]:] == -1)


def test_ctc_greedy_head_parity(small_ctx):
    cfg, W, ctx = small_ctx
    rng = np.random.default_rng(3)
    B, T, d = 4, 37, cfg["d_model"]
    enc = rng.normal(size=(B, T, d)).astype(np.float32)
    lens = np.array([37, 1, 20, 36], np.int32)
    tok, cnt, logp = gam.gam_ctc_greedy(ctx, to_torch(enc), lens, want_logp=True)
    tok, cnt, logp = tok.cpu().numpy(), cnt.cpu().numpy(), logp.cpu().numpy()
    for b in range(B):
        z, lp, a = oracle.ctc_head(enc[b, :lens[b]].astype(np.float64), W)
        assert max_abs(logp[b, :lens[b]], lp) < 1e-4
        assert np.all(logp[b, lens[b]:] == 0)
        zs = np.sort(z, axis=1)
        clear = (zs[:, -1] - zs[:, -2]) > 1e-3
        ref = oracle.greedy_collapse(a, cfg["n_classes"] - 1)
        if clear.all():
            assert tok[b, :cnt[b]].tolist() == ref


@pytest.mark.parametrize("precision,C", [("fp16", 34), ("fp16", 257), ("int8_g64", 257), ("int6_g64", 257),
                                         ("int4_g64", 34)])
def test_ctc_greedy_tensor_core_head(precision, C):
    """fp16 / INT8 contexts run the head on tensor cores with the fp32 frames
    split into fp16 hi + lo parts, so the activations keep ~22 bits.  fp16
    weights are exact: log-probs within 1e-4 of the oracle.  INT8 weights are
    dequantised in the mainloop and q*s is rounded once to fp16 (rms relative
    error 2^-11/sqrt(3) ~ 2.8e-4 per weight): here |z| ~ sqrt(256) * 0.02 = 0.32,
    so the logit error has sigma ~ 9e-5 and its maximum over the 38k values of
    this test stays below ~5 sigma: bound 1e-3 for INT8.  The 6- and 4-bit weights
    are dequantised the same way (one fp16 rounding of q*s), so the same bound holds."""
    cfg, W = config_and_weights(small_model(layers=1), C, precision)
    ctx = gam.gam_create(cfg, W, 6, 100000)
    rng = np.random.default_rng(C)
    B, T, d = 5, 150, cfg["d_model"]
    enc = rng.normal(size=(B, T, d)).astype(np.float32)
    lens = np.array([150, 0, 1, 77, 149], np.int32)
    tok, cnt, logp = gam.gam_ctc_greedy(ctx, to_torch(enc), lens, want_logp=True)
    tok, cnt, logp = tok.cpu().numpy(), cnt.cpu().numpy(), logp.cpu().numpy()
    for b in range(B):
        z, lp, a = oracle.ctc_head(enc[b, :lens[b]].astype(np.float64), W)
        assert max_abs(logp[b, :lens[b]], lp) < (1e-3 if precision.startswith("int") else 1e-4)
        assert np.all(logp[b, lens[b]:] == 0)
        zs = np.sort(z, axis=1) if lens[b] else np.zeros((0, 2))
        if np.all(zs[:, -1] - zs[:, -2] > 2e-3):
            assert tok[b, :cnt[b]].tolist() == oracle.greedy_collapse(a, C - 1)
    ctx.close()
