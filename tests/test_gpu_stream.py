"""Pseudo-streaming (gam_stream_*): every push re-recognises the last window of
the audio pushed so far ("GigaAM on MLX: the transcripts matched, but the model
was broken", "Streaming").  Each push's tokens must equal, exactly, those of
gam_encode + gam_ctc_greedy run directly on the same window of samples (the
same kernels on the same input), over pushes of ragged sizes, a push larger
than the window, empty pushes, windows too short for one encoder frame, and a
run of equal pushes on a full window where the context's CUDA graphs replay."""
import numpy as np
import pytest

from conformer_speech_recognition_b200 import gam, synth
from gpu_common import config_and_weights, small_model, to_torch

pytestmark = pytest.mark.gpu


def _direct(ctx, window):
    audio = window[None, :].astype(np.float32)
    lens = np.array([len(window)], np.int32)
    enc, el = gam.gam_encode(ctx, to_torch(audio), lens)
    tok, cnt, _ = gam.gam_ctc_greedy(ctx, enc, el)
    return tok.cpu().numpy()[0, :int(cnt.cpu().numpy()[0])]


def test_stream_matches_direct_window():
    cfg, W = config_and_weights(small_model(layers=2), 34, "fp16")
    window = 3 * 16000
    ctx = gam.gam_create(cfg, W, 1, window)
    st = gam.Stream(ctx, window)
    audio, _ = synth.random_audio([220000], seed=31)
    x = audio[0]
    sizes = [100, 1000, 0, 5920, 8000, 16000, 1, 37123, 70000, 4000, 0] + [8000] * 8
    assert sum(sizes) <= len(x)
    pos = 0
    direct_ctx = gam.gam_create(cfg, W, 1, window)  # a second context: its graphs never see the stream's pointers
    for n in sizes:
        tok, start = st.push(x[pos:pos + n])
        pos += n
        lo = max(0, pos - window)
        assert start == lo
        win = x[lo:pos]
        if len(win) < 1280:
            assert len(tok) == 0
            continue
        ref = _direct(direct_ctx, win)
        assert tok.tolist() == ref.tolist(), (pos, len(win))
    st.reset()
    tok, start = st.push(x[:16000])
    assert start == 0 and tok.tolist() == _direct(direct_ctx, x[:16000]).tolist()
    st.close()
    gam.gam_device_status(ctx)
    ctx.close()
    direct_ctx.close()


def test_stream_window_above_capacity_rejected():
    cfg, W = config_and_weights(small_model(layers=1), 34, "fp16")
    ctx = gam.gam_create(cfg, W, 1, 32000)
    with pytest.raises(gam.GamError) as e:
        gam.Stream(ctx, 64000)
    assert e.value.name == "GAM_ERR_CAPACITY"
    ctx.close()
