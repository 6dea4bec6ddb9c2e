"""Failure handling through the C ABI on a GPU context: bad arguments, capacity
overflow, short clips, missing / misshaped weights and an injected CUDA error
(all made on the host), and a bounded device wait that runs out (a pipeline
stage that is never filled; the kernel gives up after 1 ms and returns).  No
test here faults, traps or hangs the GPU."""
import numpy as np
import pytest

from conformer_speech_recognition_b200 import gam, synth
from gpu_common import config_and_weights, small_model, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx_small():
    cfg, W = config_and_weights(small_model(layers=1), 34, "fp16")
    ctx = gam.gam_create(cfg, W, 2, 32000)
    yield cfg, W, ctx
    ctx.close()


def test_capacity_and_shape_errors(ctx_small):
    cfg, W, ctx = ctx_small
    audio, lens = synth.random_audio([16000, 16000, 16000], seed=1)
    with pytest.raises(gam.GamError) as e:
        gam.gam_encode(ctx, to_torch(audio), lens)
    assert e.value.name == "GAM_ERR_CAPACITY"
    audio, lens = synth.random_audio([40000], seed=1)
    with pytest.raises(gam.GamError) as e:
        gam.gam_encode(ctx, to_torch(audio), lens)
    assert e.value.name == "GAM_ERR_CAPACITY"
    audio, lens = synth.random_audio([16000, 1279], seed=1)
    with pytest.raises(gam.GamError) as e:
        gam.gam_encode(ctx, to_torch(audio), lens)
    assert e.value.name == "GAM_ERR_SHAPE"
    with pytest.raises(gam.GamError) as e:
        gam.gam_encode_stage(ctx, to_torch(audio), np.array([16000, 16000], np.int32), 5, 1)
    assert e.value.name == "GAM_ERR_INVALID_ARG"


def test_weight_errors():
    cfg, W = config_and_weights(small_model(layers=1), 34, "fp16")
    W2 = dict(W)
    del W2["layers.0.attn.linear_k.weight"]
    with pytest.raises(gam.GamError) as e:
        gam.gam_create(cfg, W2, 1, 16000)
    assert e.value.name == "GAM_ERR_WEIGHTS" and "linear_k" in str(e.value)
    W3 = dict(W)
    W3["layers.0.conv.depthwise.weight"] = np.zeros((256, 1, 7), np.float16)
    with pytest.raises(gam.GamError) as e:
        gam.gam_create(cfg, W3, 1, 16000)
    assert e.value.name == "GAM_ERR_WEIGHTS"


def test_injected_cuda_error_then_recovery(ctx_small):
    cfg, W, ctx = ctx_small
    audio, lens = synth.random_audio([16000], seed=2)
    a = to_torch(audio)
    ref, _ = gam.gam_encode(ctx, a, lens)
    gam.gam_debug_inject_cuda_error(ctx, 2, 1)  # cudaErrorMemoryAllocation, reported by the next check
    with pytest.raises(gam.GamError) as e:
        gam.gam_encode(ctx, a, lens)
    assert e.value.name == "GAM_ERR_CUDA"
    again, _ = gam.gam_encode(ctx, a, lens)
    assert np.array_equal(again.cpu().numpy(), ref.cpu().numpy())
    gam.gam_device_status(ctx)


def test_bounded_wait_runs_out_and_context_recovers(ctx_small):
    """One GEMM tile whose second k-block is never loaded: the MMA issuer's wait
    gives up after 1 ms, the kernel drains and returns, the status word reports
    the timeout, and the next GEMM on the same context is correct."""
    import torch
    cfg, W, ctx = ctx_small
    gam.gam_device_status(ctx)
    g = torch.Generator().manual_seed(5)
    M, N, K = 128, 256, 128
    a = (torch.randn(M, K, generator=g) * 0.5).half().cuda()
    w = (torch.randn(N, K, generator=g) * 0.5).half().cuda()
    bias = torch.randn(N, generator=g).float().cuda()
    out = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    gam.gam_debug_wait_timeout(ctx, 1_000_000, 1)
    gam.gam_debug_gemm(ctx, 2, a, w, bias, out)
    torch.cuda.synchronize()
    with pytest.raises(gam.GamError) as e:
        gam.gam_device_status(ctx)
    assert e.value.name == "GAM_ERR_DEVICE_TIMEOUT"
    gam.gam_profile_reset(ctx)          # clears the status word
    gam.gam_device_status(ctx)
    out.zero_()
    gam.gam_debug_gemm(ctx, 2, a, w, bias, out)
    torch.cuda.synchronize()
    ref = a.float() @ w.float().T + bias
    assert torch.allclose(out, ref, rtol=1e-3, atol=1e-3)
    gam.gam_device_status(ctx)
