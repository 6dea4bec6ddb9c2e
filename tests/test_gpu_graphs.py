"""CUDA-graph replay of repeated calls (gam_graphs_enable): the first call with a
given (lengths, pointers) runs eagerly, the second is captured, later ones replay.
Every variant must give bit-identical results to eager execution, read the
current contents of its buffers, and never reuse a graph for other lengths."""
import numpy as np
import pytest
import torch

from conformer_speech_recognition_b200 import gam, synth
from gpu_common import config_and_weights, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def model():
    cfg, W = config_and_weights(dict(synth.V3, n_layers=2), 34, "fp16")
    return cfg, W


def _eager(cfg, W, audio, lens):
    ctx = gam.gam_create(cfg, W, 4, 48000)
    gam.gam_graphs_enable(ctx, False)
    enc, el = gam.gam_encode(ctx, audio, lens)
    tok, cnt, _ = gam.gam_ctc_greedy(ctx, enc, el)
    torch.cuda.synchronize()
    out = enc.cpu().numpy(), tok.cpu().numpy(), cnt.cpu().numpy()
    ctx.close()
    return out


def test_replay_matches_eager_and_reads_new_contents(model):
    cfg, W = model
    lens = [16000, 47000, 23456]
    audio_np, _ = synth.random_audio(lens, seed=31)
    audio = to_torch(np.pad(audio_np, ((0, 0), (0, 48000 - audio_np.shape[1]))))
    ref_enc, ref_tok, ref_cnt = _eager(cfg, W, audio, lens)
    ctx = gam.gam_create(cfg, W, 4, 48000)
    _, el, _, tmax = gam.gam_plan_lengths(cfg, lens)
    enc = torch.empty((3, tmax, cfg["d_model"]), dtype=torch.float32, device="cuda")
    tok = torch.empty((3, tmax), dtype=torch.int32, device="cuda")
    cnt = torch.empty((3,), dtype=torch.int32, device="cuda")
    for call in range(4):  # eager, capture + launch, replay, replay
        enc.fill_(float("nan"))
        tok.fill_(-7)
        gam.gam_encode(ctx, audio, lens, out=enc)
        gam.gam_ctc_greedy(ctx, enc, el, tokens=tok, counts=cnt)
        torch.cuda.synchronize()
        assert np.array_equal(enc.cpu().numpy(), ref_enc), call
        assert np.array_equal(tok.cpu().numpy(), ref_tok), call
        assert np.array_equal(cnt.cpu().numpy(), ref_cnt), call
    # same pointers, new audio: the replay reads the buffer's current contents
    audio_np2, _ = synth.random_audio(lens, seed=32)
    audio.copy_(to_torch(np.pad(audio_np2, ((0, 0), (0, 48000 - audio_np2.shape[1])))))
    ref2 = _eager(cfg, W, audio, lens)
    gam.gam_encode(ctx, audio, lens, out=enc)
    gam.gam_ctc_greedy(ctx, enc, el, tokens=tok, counts=cnt)
    torch.cuda.synchronize()
    assert np.array_equal(enc.cpu().numpy(), ref2[0])
    assert np.array_equal(cnt.cpu().numpy(), ref2[2])
    assert not np.array_equal(ref2[0], ref_enc)
    gam.gam_device_status(ctx)
    ctx.close()


def test_other_lengths_get_their_own_graph(model):
    cfg, W = model
    a_np, _ = synth.random_audio([48000, 48000, 48000], seed=33)
    audio = to_torch(a_np)
    ctx = gam.gam_create(cfg, W, 4, 48000)
    outs = {}
    for lens in ([48000, 30000, 20000], [20000, 48000, 30000], [48000, 30000, 20000], [20000, 48000, 30000]):
        _, el, _, tmax = gam.gam_plan_lengths(cfg, lens)
        out = outs.setdefault(tuple(lens), torch.empty((3, tmax, cfg["d_model"]), dtype=torch.float32, device="cuda"))
        for _ in range(3):  # reach the replay path for this key
            out.fill_(float("nan"))
            gam.gam_encode(ctx, audio, lens, out=out)
        torch.cuda.synchronize()
        ref = _eager(cfg, W, audio, lens)[0]
        got = out.cpu().numpy()
        for i in range(3):
            assert np.array_equal(got[i, :el[i]], ref[i, :el[i]]), (lens, i)
    ctx.close()


def test_transcribe_repeats_match(model):
    cfg, W = model
    lens = [16000, 40000]
    a_np, _ = synth.random_audio(lens, seed=34)
    host = torch.from_numpy(np.ascontiguousarray(a_np)).pin_memory()
    ctx = gam.gam_create(cfg, W, 4, 48000)
    _, _, _, tmax = gam.gam_plan_lengths(cfg, lens)
    tok_h = torch.empty((2, tmax), dtype=torch.int32).pin_memory()
    cnt_h = torch.empty((2,), dtype=torch.int32).pin_memory()
    results = []
    for _ in range(4):
        gam.gam_transcribe(ctx, host, lens, tok_h, cnt_h)
        results.append((tok_h.numpy().copy(), cnt_h.numpy().copy()))
    for t, c in results[1:]:
        assert np.array_equal(c, results[0][1])
        for i in range(2):
            assert np.array_equal(t[i, :c[i]], results[0][0][i, :c[i]])
    ctx.close()


def test_more_keys_than_graph_slots(model):
    """20 call keys against 16 table slots, called round-robin four times with
    fresh audio each round: eager, captured (the last four evict the first four),
    replayed or eager again, then the first four recaptured into slots whose last
    replay may still be queued.  Every call must equal an eager run bit for bit."""
    cfg, W = model
    cfg = dict(cfg, n_layers=1)
    W = {k: v for k, v in W.items() if not k.startswith("layers.") or k.startswith("layers.0.")}
    n_keys = 20
    lens_of = [[16000 + 1280 * k] for k in range(n_keys)]
    ctx = gam.gam_create(cfg, W, 1, 48000)
    eager = gam.gam_create(cfg, W, 1, 48000)
    gam.gam_graphs_enable(eager, False)
    outs = []
    for lens in lens_of:
        _, el, _, tmax = gam.gam_plan_lengths(cfg, lens)
        outs.append(torch.empty((1, tmax, cfg["d_model"]), dtype=torch.float32, device="cuda"))
    audio = torch.empty((1, 48000), dtype=torch.float32, device="cuda")
    for rnd in range(4):
        for k, lens in enumerate(lens_of):
            a_np, _ = synth.random_audio([48000], seed=1000 * rnd + k)
            audio.copy_(to_torch(a_np))
            outs[k].fill_(float("nan"))
            gam.gam_encode(ctx, audio, lens, out=outs[k])
            ref, el = gam.gam_encode(eager, audio, lens)
            torch.cuda.synchronize()
            assert np.array_equal(outs[k].cpu().numpy()[0, :el[0]], ref.cpu().numpy()[0, :el[0]]), (rnd, k)
    gam.gam_device_status(ctx)
    ctx.close()
    eager.close()
