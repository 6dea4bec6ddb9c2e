"""gam_ctc_collapse_noalloc: greedy decoding for callers that cannot allocate
device memory (no context, scratch in a fixed device array).  Its tokens and
counts must equal gam_ctc_collapse's on the same logits, exactly (the collapse
is integer work), on two calls in a row, so that the second call sees the
scratch the first one left behind; and both must equal the oracle's collapse
of numpy's argmax of the same logits.  One case runs without creating any
context.  This file is collected last."""
import numpy as np
import pytest

import oracle
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
    z[:, 4::17, :] = -np.inf          # frames of all -inf: index 0, as numpy's argmax
    z[:, 6::19, 5 % C] = np.nan       # a NaN ranks above every number
    z[:, 6::19, 7 % C] = np.nan       # (the first NaN wins)
    return z


def _oracle_tokens(z, lens, C):
    out = []
    for b in range(z.shape[0]):
        a = np.argmax(z[b, :lens[b]], axis=1) if lens[b] else np.zeros(0, np.int64)
        out.append(oracle.greedy_collapse(a, C - 1))
    return out


def _check_against_oracle(tok, cnt, z, lens, C):
    tok, cnt = tok.cpu().numpy(), cnt.cpu().numpy()
    for b, ref in enumerate(_oracle_tokens(z, lens, C)):
        assert cnt[b] == len(ref), b
        assert tok[b, :cnt[b]].tolist() == ref, b
        assert np.all(tok[b, cnt[b]:] == -1), b


def test_noalloc_without_any_context():
    """No gam_ctx is created in this test: the call needs none."""
    import torch
    rng = np.random.default_rng(7)
    B, T, C = 4, 200, 34
    lens = np.array([200, 1, 0, 123], np.int32)
    z_np = _logits(rng, B, T, C)
    z = torch.from_numpy(z_np).cuda()
    lens_dev = torch.from_numpy(lens).cuda()
    for _ in range(2):
        tok = torch.full((B, T), 777, dtype=torch.int32, device="cuda")
        cnt = torch.full((B,), 777, dtype=torch.int32, device="cuda")
        gam.gam_ctc_collapse_noalloc(z, lens_dev, tok, cnt)
        torch.cuda.synchronize()
        _check_against_oracle(tok, cnt, z_np, lens, C)


def test_noalloc_matches_collapse_two_calls():
    import torch
    cfg, W = config_and_weights(small_model(layers=1), 34, "fp16")
    ctx = gam.gam_create(cfg, W, 8, 200000)
    rng = np.random.default_rng(2024)
    cases = [(6, 300, 34, [300, 0, 1, 299, 150, 17]), (3, 257, 257, [257, 200, 3])]
    for B, T, C, lens in cases:
        z_np = _logits(rng, B, T, C)
        z = torch.from_numpy(z_np).cuda()
        lens = np.array(lens, np.int32)
        ref_tok, ref_cnt = gam.gam_ctc_collapse(ctx, z, lens)
        torch.cuda.synchronize()
        _check_against_oracle(ref_tok, ref_cnt, z_np, lens, C)
        lens_dev = torch.from_numpy(lens).cuda()
        for _ in range(2):
            tok = torch.full((B, T), 12345, dtype=torch.int32, device="cuda")
            cnt = torch.full((B,), 12345, dtype=torch.int32, device="cuda")
            gam.gam_ctc_collapse_noalloc(z, lens_dev, tok, cnt)
            torch.cuda.synchronize()
            assert torch.equal(cnt, ref_cnt)
            assert torch.equal(tok, ref_tok)
            _check_against_oracle(tok, cnt, z_np, lens, C)
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
