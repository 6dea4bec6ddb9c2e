"""Every call writes inside its documented output extent and nowhere else: each
output buffer is the front of a larger allocation whose tail holds a canary
pattern, and the tail must be intact after the call (a device-side stand-in for
a bounds checker, which is not available here)."""
import numpy as np
import pytest

from conformer_speech_recognition_b200 import gam, synth
from gpu_common import config_and_weights, small_model, to_torch

pytestmark = pytest.mark.gpu

PAD = 4096
CANARY_F = -12345.678
CANARY_I = -77777


def _padded(shape, dtype):
    import torch
    n = int(np.prod(shape))
    fill = CANARY_F if dtype == torch.float32 else CANARY_I
    buf = torch.full((n + PAD,), fill, dtype=dtype, device="cuda")
    return buf, buf[:n].view(*shape)


def _tail_intact(buf, n):
    import torch
    torch.cuda.synchronize()
    t = buf[n:].cpu().numpy()
    ref = CANARY_F if t.dtype == np.float32 else CANARY_I
    return bool(np.all(t == ref))


@pytest.mark.parametrize("precision", ["fp16", "int4_g64", "fp32"])
def test_outputs_stay_in_bounds(precision):
    import torch
    cfg, W = config_and_weights(small_model(layers=1), 34, precision)
    lengths = [16000, 1280, 23456]
    audio, lens = synth.random_audio(lengths, seed=3)
    ctx = gam.gam_create(cfg, W, 3, 24000)
    fr, el, fmax, tmax = gam.gam_plan_lengths(cfg, lens)
    B, d = len(lens), cfg["d_model"]
    a = to_torch(audio)

    mb, mel = _padded((B, fmax, 64), torch.float32)
    gam.gam_logmel(ctx, a, lens, out=mel)
    assert _tail_intact(mb, mel.numel())

    eb, enc = _padded((B, tmax, d), torch.float32)
    gam.gam_encode(ctx, a, lens, out=enc)
    assert _tail_intact(eb, enc.numel())

    tb, tok = _padded((B, tmax), torch.int32)
    cb, cnt = _padded((B,), torch.int32)
    lb, logp = _padded((B, tmax, cfg["n_classes"]), torch.float32)
    gam.gam_ctc_greedy(ctx, enc, el, tokens=tok, counts=cnt, logp=logp)
    assert _tail_intact(tb, tok.numel()) and _tail_intact(cb, cnt.numel()) and _tail_intact(lb, logp.numel())

    tb2, tok2 = _padded((B, tmax), torch.int32)
    fb2, frm2 = _padded((B, tmax), torch.int32)
    cb2, cnt2 = _padded((B,), torch.int32)
    gam.gam_ctc_greedy_frames(ctx, enc, el, tokens=tok2, frames=frm2, counts=cnt2)
    assert _tail_intact(tb2, tok2.numel()) and _tail_intact(fb2, frm2.numel()) and _tail_intact(cb2, cnt2.numel())

    gam.gam_rnnt_attach(ctx, dict(n_classes=34, max_symbols=4), synth.random_rnnt_weights(d, 34))
    mt = 7
    tb3, tok3 = _padded((B, mt), torch.int32)
    fb3, frm3 = _padded((B, mt), torch.int32)
    cb3, cnt3 = _padded((B,), torch.int32)
    gam.gam_rnnt_greedy(ctx, enc, el, max_tokens=mt, tokens=tok3, frames=frm3, counts=cnt3)
    assert _tail_intact(tb3, tok3.numel()) and _tail_intact(fb3, frm3.numel()) and _tail_intact(cb3, cnt3.numel())
    gam.gam_device_status(ctx)
    ctx.close()
