"""Unit parity of the encoder's GEMM kernels through the C ABI (gam_debug_gemm):
out += A . W^T + bias with fp16 operands and fp32 accumulation, for the
tensor-core (tcgen05) and CUDA-core implementations, against NumPy in fp64.
impl 0 lets the library choose the tile shape, 2 forces single-CTA tiles,
3 paired-CTA (cta_group::2) tiles and 4 K split over a cluster; a tile width
(128, 192, 256) shifted left by 8 bits forces the width too."""
import numpy as np
import pytest

from conformer_speech_recognition_b200 import gam
from gpu_common import config_and_weights, small_model

pytestmark = pytest.mark.gpu

# fp32 accumulation of K fp16 products: relative to the largest output
TOL_GEMM_REL = 2e-4


@pytest.fixture(scope="module")
def ctx():
    cfg, W = config_and_weights(small_model(layers=1), 34, "fp16")
    c = gam.gam_create(cfg, W, 1, 16000)
    yield c
    c.close()


@pytest.mark.parametrize("impl", [0, 1, 2, 3], ids=["tcgen05", "cuda_cores", "tc_single_cta", "tc_cta_pair"])
@pytest.mark.parametrize("M,N,K,lda", [(128, 256, 64, 64), (300, 512, 320, 320), (1000, 768, 768, 768),
                                       (5000, 3072, 768, 768), (2100, 256, 3072, 3072),
                                       (777, 768, 320, 128)],
                         ids=["one_tile", "ragged_m", "d768", "many_tiles", "deep_k", "strided_view"])
def test_gemm_parity(ctx, impl, M, N, K, lda):
    import torch
    rng = np.random.default_rng(M + N + K)
    rows_needed = (M - 1) * lda + K if lda >= K else (M + 2) * lda
    flat = rng.normal(size=rows_needed).astype(np.float16)
    A = np.lib.stride_tricks.as_strided(flat, shape=(M, K), strides=(lda * 2, 2))
    Wt = rng.normal(size=(N, K)).astype(np.float16)
    b = rng.normal(size=N).astype(np.float32)
    out0 = rng.normal(size=(M, N)).astype(np.float32)
    ta = torch.from_numpy(flat).cuda()
    a_view = torch.as_strided(ta, (M, K), (lda, 1))
    tw = torch.from_numpy(Wt).cuda()
    tb = torch.from_numpy(b).cuda()
    to = torch.from_numpy(out0.copy()).cuda()
    gam.gam_debug_gemm(ctx, impl, a_view, tw, tb, to)
    got = to.cpu().numpy()
    ref = out0.astype(np.float64) + A.astype(np.float64) @ Wt.astype(np.float64).T + b
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err <= TOL_GEMM_REL, err
    gam.gam_device_status(ctx)


@pytest.mark.parametrize("M,N,K", [(300, 768, 768), (9000, 768, 3072), (4000, 2304, 768), (1200, 1024, 1024)],
                         ids=["bn192_small", "bn192_deep", "qkv_width", "bn128_d1024"])
def test_gemm_tile_widths(ctx, M, N, K):
    """Shapes for which the tensor-core GEMM picks a 192- or 128-column tile."""
    test_gemm_parity(ctx, 0, M, N, K, K)


@pytest.mark.parametrize("M,N,K,lda", [(129, 768, 64, 64), (256, 768, 128, 128), (20000, 1536, 768, 768),
                                       (4097, 768, 3072, 3072), (3001, 768, 1536, 768)],
                         ids=["peer_rows_empty", "one_pair_row", "more_tiles_than_pairs", "deep_k_ragged",
                              "strided_view_wide"])
@pytest.mark.parametrize("kind", [2, 3], ids=["single_cta", "cta_pair"])
@pytest.mark.parametrize("width", [128, 192, 256])
def test_gemm_tile_shapes(ctx, M, N, K, lda, kind, width):
    """Every tile shape: a pair whose second CTA holds only padding rows, a single
    row of pair tiles, more tiles than co-resident pairs, a deep ragged K loop and
    the convolution view, at each tile width."""
    test_gemm_parity(ctx, kind | (width << 8), M, N, K, lda)


@pytest.mark.parametrize("M,N,K", [(24, 768, 768), (128, 3072, 768), (200, 768, 3072), (256, 2304, 768)],
                         ids=["batch1_rows", "one_m_block", "deep_k", "two_m_blocks"])
def test_gemm_narrow_tiles_few_rows(ctx, M, N, K):
    """64-column single-CTA tiles, which the library picks for GEMMs of at most
    256 rows; forced and chosen."""
    test_gemm_parity(ctx, 2 | (64 << 8), M, N, K, K)
    test_gemm_parity(ctx, 0, M, N, K, K)


def test_gemm_width_must_divide_n(ctx):
    import torch
    a = torch.zeros(256, 64, dtype=torch.float16, device="cuda")
    w = torch.zeros(1024, 64, dtype=torch.float16, device="cuda")
    b = torch.zeros(1024, dtype=torch.float32, device="cuda")
    o = torch.zeros(256, 1024, dtype=torch.float32, device="cuda")
    with pytest.raises(gam.GamError, match="SHAPE|shape"):
        gam.gam_debug_gemm(ctx, 3 | (192 << 8), a, w, b, o)
    with pytest.raises(gam.GamError):
        gam.gam_debug_gemm(ctx, 3 | (100 << 8), a, w, b, o)


@pytest.mark.parametrize("M,N,K", [(24, 768, 3072), (25, 768, 768), (200, 3072, 768), (129, 2304, 768),
                                   (256, 768, 1536), (1, 256, 512)],
                         ids=["batch1_ffn_down", "batch1_out_proj", "ffn_up_two_m_blocks", "qkv_ragged",
                              "two_full_m_blocks", "one_row"])
def test_gemm_split_k(ctx, M, N, K):
    """K split over a cluster of 2 to 4 CTAs, the leader adding the partial sums
    in rank order: forced (kind 4) and as the library chooses for few rows."""
    test_gemm_parity(ctx, 4, M, N, K, K)
    test_gemm_parity(ctx, 0, M, N, K, K)
