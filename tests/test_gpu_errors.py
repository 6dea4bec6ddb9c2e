"""Failure handling through the C ABI on a GPU context, all made on the host:
bad arguments, capacity overflow, short clips, missing / misshaped weights and
an injected CUDA error.  No test here faults, traps or hangs the GPU."""
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
