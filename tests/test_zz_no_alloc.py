"""gam_ctc_collapse_noalloc: greedy decoding for callers that cannot allocate
device memory (no context, scratch in a fixed device array).  Its tokens and
counts must equal gam_ctc_collapse's on the same logits, exactly (the collapse
is integer work), on two calls in a row, so that the second call sees the
scratch the first one left behind.  This file is collected last."""
import numpy as np
import pytest

from conformer_speech_recognition_b200 import gam
from gpu_common import config_and_weights, small_model

pytestmark = pytest.mark.gpu


def _logits(rng, B, T, C):
    z = rng.normal(size=(B, T, C)).astype(np.float32)
    z[:, ::5, C - 1] += 8.0           # blank runs
    z[:, 1::7, 3 % C] += 9.0          # repeats of one symbol
    m = z[:, 2::11].max(axis=2) + 1.0
    z[:, 2::11, 1] = m                # exact ties: the lowest index wins
    z[:, 2::11, 2] = m
    return z


def test_noalloc_matches_collapse_two_calls():
    import torch
    cfg, W = config_and_weights(small_model(layers=1), 34, "fp16")
    ctx = gam.gam_create(cfg, W, 8, 200000)
    rng = np.random.default_rng(2024)
    cases = [(6, 300, 34, [300, 0, 1, 299, 150, 17]), (3, 257, 257, [257, 200, 3])]
    for B, T, C, lens in cases:
        z = torch.from_numpy(_logits(rng, B, T, C)).cuda()
        lens = np.array(lens, np.int32)
        ref_tok, ref_cnt = gam.gam_ctc_collapse(ctx, z, lens)
        lens_dev = torch.from_numpy(lens).cuda()
        for _ in range(2):
            tok = torch.full((B, T), 12345, dtype=torch.int32, device="cuda")
            cnt = torch.full((B,), 12345, dtype=torch.int32, device="cuda")
            gam.gam_ctc_collapse_noalloc(z, lens_dev, tok, cnt)
            torch.cuda.synchronize()
            assert torch.equal(cnt, ref_cnt)
            assert torch.equal(tok, ref_tok)
    ctx.close()


def test_noalloc_rejects_oversize():
    import torch
    z = torch.zeros((1, 1, 2), dtype=torch.float32, device="cuda")
    lens = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tok = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1,), dtype=torch.int32, device="cuda")
    big = gam.GAM_NOALLOC_MAX_FRAMES + 1
    with pytest.raises(gam.GamError) as e:
        st = gam.lib().gam_ctc_collapse_noalloc(z.data_ptr(), lens.data_ptr(), big, 1, 2, tok.data_ptr(),
                                                cnt.data_ptr(), None)
        gam._check(st)
    assert e.value.name == "GAM_ERR_CAPACITY" and "frames" in str(e.value)
