"""GPU parity of the encoder (frontend -> subsampling -> Conformer blocks) and of
the whole encoder + CTC path, through the C ABI, against the oracle.

* fp32 build mode: every stage of every block within 1e-4 (max |delta|).
* fp16 / INT8 product modes: relative Frobenius <= 1e-2, max |delta| <= 5e-2,
  CTC frame argmax agreement >= 99.5%, on the benchmark workloads at full size
  (the GPU runs the whole batch in the benchmark's launch configuration, the
  oracle recomputes sampled clips one by one).
"""
import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import gam, synth
from gpu_common import (MIN_ARGMAX_AGREE, TOL_FP32_LAYER, TOL_MAX_ABS, TOL_REL_FRO, config_and_weights, max_abs,
                        oracle_clip, rel_fro, small_model, to_torch)

pytestmark = pytest.mark.gpu


def _stage_ref(dump, layer, stage):
    if stage == gam.STAGE_SUBSAMPLING:
        return dump["x0"]
    return dump["layers"][layer][stage - 1]


@pytest.mark.parametrize("model", [dict(synth.V3, n_layers=16), small_model(d=256, heads=4, ffn=512, layers=3, K=5)],
                         ids=["d768_h48_16L", "d256_h64_3L_k5"])
def test_fp32_every_stage_every_layer(model):
    cfg, W = config_and_weights(model, 34, "fp32")
    lengths = [16000, 25760, 1280]
    audio, lens = synth.random_audio(lengths, seed=11)
    ctx = gam.gam_create(cfg, W, 4, 32000)
    a = to_torch(audio)
    dumps = [oracle_clip(audio[i], lens[i], W, cfg, dump=True)[1] for i in range(len(lens))]
    _, el, _, _ = gam.gam_plan_lengths(cfg, lens)
    worst = 0.0
    checks = [(0, gam.STAGE_SUBSAMPLING)] + [(l, s) for l in range(cfg["n_layers"]) for s in range(1, 6)]
    for layer, stage in checks:
        out = gam.gam_encode_stage(ctx, a, lens, layer, stage).cpu().numpy()
        for i in range(len(lens)):
            ref = _stage_ref(dumps[i], layer, stage)
            assert out[i, :el[i]].shape == ref.shape
            err = max_abs(out[i, :el[i]], ref)
            worst = max(worst, err)
            assert err <= TOL_FP32_LAYER, (layer, stage, i, err)
            assert np.all(out[i, el[i]:] == 0)
    enc, el2 = gam.gam_encode(ctx, a, lens)
    assert list(el2) == list(el)
    ctx.close()
    print(f"fp32 worst per-stage max|delta| = {worst:.3e}")


def _batch_invariance(ctx, audio, lens, enc, el):
    """Every clip run alone gives the frames it has inside the full batch, so the
    oracle comparison of sampled clips carries over to the clips in between."""
    worst = 0.0
    for i in range(len(lens)):
        alone, el1 = gam.gam_encode(ctx, to_torch(audio[i:i + 1, :lens[i]]), lens[i:i + 1])
        assert el1[0] == el[i]
        worst = max(worst, max_abs(alone.cpu().numpy()[0, :el1[0]], enc[i, :el[i]]))
    assert worst <= 1e-5, worst
    return worst


def _product_check(name, cfg, W, ctx, audio, lens, sample, every_clip_alone=False):
    """Run the whole batch on the GPU; compare sampled clips with the oracle and,
    optionally, every clip of the batch with the same clip run alone."""
    a = to_torch(audio)
    enc, el = gam.gam_encode(ctx, a, lens)
    tok, cnt, logp = gam.gam_ctc_greedy(ctx, enc, el, want_logp=True)
    enc, tok, cnt, logp = enc.cpu().numpy(), tok.cpu().numpy(), cnt.cpu().numpy(), logp.cpu().numpy()
    agree = total = 0
    report = []
    for i in sample:
        ref = oracle.encode_clip(audio[i, :lens[i]].astype(np.float64), W, cfg, np.float64)
        got = enc[i, :el[i]]
        assert got.shape == ref.shape
        rf, ma = rel_fro(got, ref), max_abs(got, ref)
        report.append((int(i), rf, ma))
        assert rf <= TOL_REL_FRO, (name, i, rf)
        assert ma <= TOL_MAX_ABS, (name, i, ma)
        assert np.all(enc[i, el[i]:] == 0)
        z, lp, amax = oracle.ctc_head(ref, W)
        gpu_amax = np.argmax(logp[i, :el[i]], axis=1)
        agree += int((gpu_amax == amax).sum())
        total += len(amax)
    frac = agree / total
    print(name, "per-clip (clip, rel_fro, max_abs):", report, "argmax agreement", frac)
    assert frac >= MIN_ARGMAX_AGREE, (name, frac)
    if every_clip_alone:
        print(name, "batch invariance worst max|delta|", _batch_invariance(ctx, audio, lens, enc, el))
    return enc, el, tok, cnt


def test_c1_fp16_full():
    name = "c1_1s_b1_d768"
    cfg = synth.workload_config(name)
    _, W = config_and_weights(synth.V3, 34, "fp16")
    audio, lens = synth.workload_audio(name)
    ctx = gam.gam_create(cfg, W, 1, 16000)
    _product_check(name, cfg, W, ctx, audio, lens, [0])
    ctx.close()


def test_c2_fp16_full_batch_sampled():
    name = "c2_varlen_b32_d768"
    cfg = synth.workload_config(name)
    _, W = config_and_weights(synth.V3, 34, "fp16")
    audio, lens = synth.workload_audio(name)
    ctx = gam.gam_create(cfg, W, 32, 320000)
    order = np.argsort(lens)
    sample = [order[0], order[len(order) // 2], order[-1], order[1], order[-2]]
    enc, el, tok, cnt = _product_check(name, cfg, W, ctx, audio, lens, sample)
    # batch invariance: a clip alone gives the same valid frames as inside the batch
    i = order[len(order) // 2]
    alone, el1 = gam.gam_encode(ctx, to_torch(audio[i:i + 1, :lens[i]]), lens[i:i + 1])
    assert el1[0] == el[i]
    assert max_abs(alone.cpu().numpy()[0, :el1[0]], enc[i, :el[i]]) <= 1e-5
    ctx.close()


def test_c3_fp16_full_batch_sampled():
    name = "c3_20s_b64_d768"
    cfg = synth.workload_config(name)
    _, W = config_and_weights(synth.V3, 257, "fp16")
    audio, lens = synth.workload_audio(name)
    ctx = gam.gam_create(cfg, W, 64, 320000)
    _product_check(name, cfg, W, ctx, audio, lens, [0, 31, 63], every_clip_alone=True)
    ctx.close()


def test_c4_fp16_full_batch_sampled():
    name = "c4_30s_b32_d1024"
    cfg = synth.workload_config(name)
    _, W = config_and_weights(synth.LARGE, 257, "fp16")
    audio, lens = synth.workload_audio(name)
    ctx = gam.gam_create(cfg, W, 32, 480000)
    _product_check(name, cfg, W, ctx, audio, lens, [0, 16, 31], every_clip_alone=True)
    ctx.close()


@pytest.mark.parametrize("name", ["c5_300s_chunks15_d1024_int8", "c5_300s_chunks15_d1024_int6",
                                  "c5_300s_chunks15_d1024_int4"])
def test_c5_quantized_full_batch_sampled(name):
    """Long-form chunks on the d1024 encoder with 8-, 6- and 4-bit g64 weights
    dequantised in the GEMM mainloop; the oracle uses the same q * s in fp64."""
    cfg = synth.workload_config(name)
    _, W = config_and_weights(synth.LARGE, 257, cfg["precision"])
    audio, lens = synth.workload_audio(name)
    ctx = gam.gam_create(cfg, W, 15, 320000)
    _product_check(name, cfg, W, ctx, audio, lens, [0, 7, 14], every_clip_alone=True)
    ctx.close()


@pytest.mark.parametrize("form", ["1", "2"], ids=["attn_128_key_blocks", "attn_64_key_blocks"])
@pytest.mark.parametrize("K", [31, 5])
def test_attention_forms_small_model(form, K, monkeypatch):
    """Both tensor-core attention kernels (GAM_ATTN=1: 128-key blocks; the default:
    64-key blocks with scores double-buffered in TMEM) on ragged clips, d_h 64,
    against the oracle."""
    monkeypatch.setenv("GAM_ATTN", form)
    model = small_model(d=256, heads=4, ffn=512, layers=2, K=K)
    cfg, W = config_and_weights(model, 34, "fp16")
    audio, lens = synth.random_audio([48000, 17000, 30001], seed=11)
    ctx = gam.gam_create(cfg, W, 3, 48000)
    enc, el = gam.gam_encode(ctx, to_torch(audio), lens)
    enc = enc.cpu().numpy()
    for i in range(3):
        ref = oracle.encode_clip(audio[i, :lens[i]].astype(np.float64), W, cfg)
        assert rel_fro(enc[i, :el[i]], ref) <= TOL_REL_FRO, (form, i)
        assert max_abs(enc[i, :el[i]], ref) <= TOL_MAX_ABS, (form, i)
    gam.gam_device_status(ctx)
    ctx.close()


@pytest.mark.parametrize("tiles", ["m1", "m2"])
@pytest.mark.parametrize("precision", ["int8_g64", "int6_g64", "int4_g64"])
def test_quantized_small_model(precision, tiles, monkeypatch):
    """Both tile forms of the quantised mainloop: one 128-row A tile per converted
    B stage (GAM_QB_TILES=m1) and two (m2, the default)."""
    monkeypatch.setenv("GAM_QB_TILES", tiles)
    model = small_model(d=256, heads=4, ffn=512, layers=2, K=31)
    cfg, W = config_and_weights(model, 257, precision)
    audio, lens = synth.random_audio([20000, 9000], seed=5)
    ctx = gam.gam_create(cfg, W, 2, 20000)
    enc, el = gam.gam_encode(ctx, to_torch(audio), lens)
    enc = enc.cpu().numpy()
    for i in range(2):
        ref = oracle.encode_clip(audio[i, :lens[i]].astype(np.float64), W, cfg)
        assert rel_fro(enc[i, :el[i]], ref) <= TOL_REL_FRO
        assert max_abs(enc[i, :el[i]], ref) <= TOL_MAX_ABS
    ctx.close()


def test_transcribe_host_buffers_match_device_path():
    name = "c1_1s_b1_d768"
    cfg = synth.workload_config(name)
    _, W = config_and_weights(synth.V3, 34, "fp16")
    audio, lens = synth.random_audio([16000, 23456, 30000], seed=21)
    ctx = gam.gam_create(cfg, W, 4, 32000)
    enc, el = gam.gam_encode(ctx, to_torch(audio), lens)
    tok, cnt, _ = gam.gam_ctc_greedy(ctx, enc, el)
    tok_h, cnt_h = gam.gam_transcribe(ctx, audio, lens)
    assert np.array_equal(cnt.cpu().numpy(), cnt_h)
    assert np.array_equal(tok.cpu().numpy(), tok_h)
    ctx.close()


def test_fp32_subsampling_every_length_residue():
    """Clips of F = 7 .. 22 frames (every F mod 4 and every L' mod 8, so the
    segment layout is packed with and without slack) back to back: the
    subsampling output of each clip matches the oracle."""
    model = small_model(d=256, heads=4, ffn=512, layers=1, K=5)
    cfg, W = config_and_weights(model, 34, "fp32")
    lengths = [320 + 160 * (F - 1) + (F % 3) * 40 for F in range(7, 23)]
    audio, lens = synth.random_audio(lengths, seed=13)
    ctx = gam.gam_create(cfg, W, len(lens), int(max(lens)))
    out = gam.gam_encode_stage(ctx, to_torch(audio), lens, 0, gam.STAGE_SUBSAMPLING).cpu().numpy()
    _, el, _, _ = gam.gam_plan_lengths(cfg, lens)
    for i in range(len(lens)):
        _, dump = oracle_clip(audio[i], lens[i], W, cfg, dump=True, n_layers=0)
        assert out[i, :el[i]].shape == dump["x0"].shape
        assert max_abs(out[i, :el[i]], dump["x0"]) <= TOL_FP32_LAYER, i
    ctx.close()


def test_fp16_subsampling_tensor_core_frontend():
    """fp16 mode: tensor-core frontend (fp16 frames, DFT GEMM with the power
    epilogue, mel over the filterbank's nonzero ranges, log) and the two
    subsampling GEMMs, against the oracle's subsampling output."""
    model = small_model(d=256, heads=4, ffn=512, layers=1, K=5)
    cfg, W = config_and_weights(model, 34, "fp16")
    lengths = [1280, 16000, 37123, 320 + 160 * 40]
    audio, lens = synth.random_audio(lengths, seed=17)
    ctx = gam.gam_create(cfg, W, len(lens), int(max(lens)))
    out = gam.gam_encode_stage(ctx, to_torch(audio), lens, 0, gam.STAGE_SUBSAMPLING).cpu().numpy()
    _, el, _, _ = gam.gam_plan_lengths(cfg, lens)
    for i in range(len(lens)):
        _, dump = oracle_clip(audio[i], lens[i], W, cfg, dump=True, n_layers=0)
        got = out[i, :el[i]]
        assert got.shape == dump["x0"].shape
        assert rel_fro(got, dump["x0"]) <= TOL_REL_FRO, i
        assert max_abs(got, dump["x0"]) <= TOL_MAX_ABS, i
        assert np.all(out[i, el[i]:] == 0)
    ctx.close()
