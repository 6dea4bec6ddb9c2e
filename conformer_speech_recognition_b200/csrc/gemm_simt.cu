// CUDA-core (FFMA) GEMM with fused epilogues: C = A . B^T, fp32 accumulation.
//
// This is the fp32-precision path of every dense contraction (the tensor-core
// kernels in gemm_tc.cu serve the fp16 / INT8 products) and the path of the
// small CTC head.  A is [M, K] with an arbitrary row stride `lda`, which lets
// the two stride-2 subsampling convs run as GEMMs over a strided view of their
// input (row r reads rows 2r .. 2r+4 of a channels-last [rows, C] buffer when
// lda = 2C and K = 5C).  B is a weight in PyTorch Linear layout [N, K]: fp32,
// fp16, or INT8 with one fp16 scale per 64 consecutive K (dequantised on load).
//
// Tile 128 x 128 x 16, 256 threads, 8 x 8 outputs per thread.  A thread owns
// output columns {4 tx .. 4 tx + 3} and {64 + 4 tx .. 64 + 4 tx + 3} of its
// tile so that the value/gate pair of the GLU epilogue (weights interleaved in
// blocks of 64) sits in one thread.
#include "common.cuh"

namespace gam {
namespace {

constexpr int BM = 128, BN = 128, BK = 16;

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __half* p) { return __half2float(*p); }

template <typename T>
__device__ __forceinline__ void store_t(void* base, size_t idx, float v) {
  if constexpr (sizeof(T) == 2) reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
  else reinterpret_cast<float*>(base)[idx] = v;
}

__device__ __forceinline__ float sigmoidf_(float v) { return 1.f / (1.f + __expf(-v)); }

template <typename TA, int BT, typename TO>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const TA* __restrict__ A, const TA* __restrict__ A2, int n_split, int lda,
                 const void* __restrict__ Bw, const __half* __restrict__ Bscale, int M, int N, int K, int epi,
                 EpiParams ep) {
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const TA* Ause = (A2 != nullptr && n0 >= n_split) ? A2 : A;

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int lr = tid >> 1, lk = (tid & 1) * 8;
  for (int k0 = 0; k0 < K; k0 += BK) {
    {
      const int r = m0 + lr;
      float v[8];
      if (r < M) {
        const TA* p = Ause + (size_t)r * lda + k0 + lk;
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = ld_f(p + j);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) As[lk + j][lr] = v[j];
    }
    {
      const int n = n0 + lr;
      float v[8];
      if (n < N) {
        if constexpr (BT == 0) {
          const float* p = reinterpret_cast<const float*>(Bw) + (size_t)n * K + k0 + lk;
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = p[j];
        } else if constexpr (BT == 1) {
          const __half* p = reinterpret_cast<const __half*>(Bw) + (size_t)n * K + k0 + lk;
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = __half2float(p[j]);
        } else {
          const int8_t* p = reinterpret_cast<const int8_t*>(Bw) + (size_t)n * K + k0 + lk;
          const float s = __half2float(Bscale[(size_t)n * (K / 64) + (k0 + lk) / 64]);
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = (float)p[j] * s;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) Bs[lk + j][lr] = v[j];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[k][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[k][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  // ---- epilogue ----
  int cols[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) cols[j] = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = m0 + ty * 8 + i;
    if (r >= M) continue;
    switch (epi) {
      case EPI_SWISH:
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float v = acc[i][j] + ep.bias[cols[j]];
          store_t<TO>(ep.out, (size_t)r * ep.ldo + cols[j], v * sigmoidf_(v));
        }
        break;
      case EPI_GLU: {
        const int oc = (n0 >> 1) + tx * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float v = acc[i][j] + ep.bias[cols[j]];
          const float gt = acc[i][j + 4] + ep.bias[cols[j + 4]];
          store_t<TO>(ep.out, (size_t)r * ep.ldo + oc + j, v * sigmoidf_(gt));
        }
      } break;
      case EPI_RESID:
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float* px = ep.x + (size_t)r * ep.ldo + cols[j];
          *px += ep.alpha * (acc[i][j] + ep.bias[cols[j]]);
        }
        break;
      case EPI_QKV:
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = cols[j];
          const int which = n / ep.d_model;
          const int rem = n - which * ep.d_model;
          const int h = rem / ep.d_head, c = rem - h * ep.d_head;
          const float v = acc[i][j] + ep.bias[n];
          if (which < 2)
            store_t<TO>(ep.qk, (((size_t)which * ep.n_heads + h) * ep.rows_pad + r) * 64 + c, v);
          else
            store_t<TO>(ep.vt, ((size_t)h * 64 + c) * ep.rows_pad + r, v);
        }
        break;
      case EPI_CONV1: {
        const int ci = ep.clips.find(r, 2, 2);
        const int t = r - (2 * ep.clips.e(ci) + 2);
        const bool valid = t >= 0 && t < ep.clips.L1(ci);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float v = valid ? fmaxf(acc[i][j] + ep.bias[cols[j]], 0.f) : 0.f;
          store_t<TO>(ep.out, (size_t)r * ep.ldo + cols[j], v);
        }
      } break;
      case EPI_CONV2: {
        const int ci = ep.clips.find(r, 1, 0);
        const int t = r - ep.clips.e(ci);
        const bool valid = t >= 0 && t < ep.clips.L2(ci);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float v = valid ? fmaxf(acc[i][j] + ep.bias[cols[j]], 0.f) : 0.f;
          ep.x[(size_t)r * ep.ldo + cols[j]] = v;
        }
      } break;
      case EPI_F32:
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (cols[j] < N)
            reinterpret_cast<float*>(ep.out)[(size_t)r * ep.ldo + cols[j]] = acc[i][j] + ep.bias[cols[j]];
        break;
    }
  }
}

template <typename TA, int BT>
cudaError_t launch_t(const void* A, const void* A2, int n_split, int lda, WeightOp B, int M, int N, int K,
                     int epi, int out_half, const EpiParams& ep, cudaStream_t s) {
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  if (out_half)
    gemm_simt_kernel<TA, BT, __half><<<grid, 256, 0, s>>>(
        reinterpret_cast<const TA*>(A), reinterpret_cast<const TA*>(A2), n_split, lda, B.w, B.scale, M, N, K,
        epi, ep);
  else
    gemm_simt_kernel<TA, BT, float><<<grid, 256, 0, s>>>(
        reinterpret_cast<const TA*>(A), reinterpret_cast<const TA*>(A2), n_split, lda, B.w, B.scale, M, N, K,
        epi, ep);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_simt(int a_dtype, const void* A, const void* A2, int n_split, int lda, WeightOp B, int M,
                             int N, int K, int epi, int out_half, const EpiParams& ep, cudaStream_t s) {
  if (K % BK != 0 || M <= 0 || N <= 0) return cudaErrorInvalidValue;
  if ((epi == EPI_GLU || epi == EPI_QKV || epi == EPI_SWISH || epi == EPI_RESID || epi == EPI_CONV1 ||
       epi == EPI_CONV2) && N % BN != 0)
    return cudaErrorInvalidValue;
  if (a_dtype == 0) {
    if (B.dtype == 0) return launch_t<float, 0>(A, A2, n_split, lda, B, M, N, K, epi, out_half, ep, s);
    if (B.dtype == 1) return launch_t<float, 1>(A, A2, n_split, lda, B, M, N, K, epi, out_half, ep, s);
    return launch_t<float, 2>(A, A2, n_split, lda, B, M, N, K, epi, out_half, ep, s);
  }
  if (B.dtype == 1) return launch_t<__half, 1>(A, A2, n_split, lda, B, M, N, K, epi, out_half, ep, s);
  if (B.dtype == 2) return launch_t<__half, 2>(A, A2, n_split, lda, B, M, N, K, epi, out_half, ep, s);
  return cudaErrorInvalidValue;
}

}  // namespace gam
