// Masked multi-head self-attention on CUDA cores (fp32 math), online softmax.
//
// softmax(Q K^T / sqrt(d_head) + mask) V per (clip, head), keys at or beyond
// the clip's valid length L' masked out ("GigaAM MLX port for Mac", "What is
// inside the model": masking is part of the reproduced path).  Q and K come
// head-major [2][H][rows][64] (head dim padded to 64), V transposed
// [H][64][rows], output O [rows, d] in the activation type.
//
// CTA = 64 queries of one (clip, head); 256 threads, 4 per query row.  The
// query row lives in registers (pre-scaled by log2(e)/sqrt(d_head) so the
// softmax uses exp2); each KV block of 64 keys is staged in shared memory.
#include "common.cuh"

namespace gam {
namespace {

constexpr int BQ = 64, BKV = 64;
constexpr int KS = 65;  // padded row stride of the K / P tiles
constexpr size_t SMEM = (size_t)(BKV * KS + BKV * KS + BQ * KS) * sizeof(float);

__device__ __forceinline__ float ldv(const float* p) { return *p; }
__device__ __forceinline__ float ldv(const __half* p) { return __half2float(*p); }

template <typename T>
__global__ void __launch_bounds__(256)
attn_simt_kernel(const T* __restrict__ qk, const T* __restrict__ vt, Clips clips, T* __restrict__ o, int rows_pad,
                 int H, int dh, float qscale) {
  extern __shared__ float sm[];
  float* Ks = sm;                 // [BKV][KS]
  float* Vs = Ks + BKV * KS;      // [BKV][KS]
  float* Ps = Vs + BKV * KS;      // [BQ][KS]
  const int b = blockIdx.z, h = blockIdx.y;
  const int L = clips.L2(b), e0 = clips.e(b);
  const int q0 = blockIdx.x * BQ;
  if (q0 >= L) return;
  const int tid = threadIdx.x, r = tid >> 2, qd = tid & 3;
  const int d = H * dh;

  float qv[64];
  const int qrow = e0 + q0 + r;
  const T* qp = qk + (((size_t)0 * H + h) * rows_pad + min(qrow, rows_pad - 1)) * 64;
#pragma unroll
  for (int c = 0; c < 64; ++c) qv[c] = c < dh ? ldv(qp + c) * qscale : 0.f;

  float acc[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) acc[m] = 0.f;
  float mrow = -INFINITY, lrow = 0.f;

  const T* kbase = qk + ((size_t)1 * H + h) * rows_pad * 64;
  const T* vbase = vt + (size_t)h * 64 * rows_pad;
  for (int k0 = 0; k0 < L; k0 += BKV) {
    for (int idx = tid; idx < BKV * 64; idx += 256) {
      const int j = idx >> 6, c = idx & 63;
      const int kr = e0 + k0 + j;
      Ks[j * KS + c] = (kr < rows_pad) ? ldv(kbase + (size_t)kr * 64 + c) : 0.f;
      const int c2 = idx / BKV, j2 = idx % BKV;  // V^T: consecutive threads walk keys
      const int vr = e0 + k0 + j2;
      Vs[j2 * KS + c2] = (vr < rows_pad) ? ldv(vbase + (size_t)c2 * rows_pad + vr) : 0.f;
    }
    __syncthreads();
    float s[16];
    float mloc = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const int key = jj * 4 + qd;
      const float* kr = Ks + key * KS;
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (c < dh) a = fmaf(qv[c], kr[c], a);
      s[jj] = (k0 + key < L) ? a : -INFINITY;
      mloc = fmaxf(mloc, s[jj]);
    }
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const float mnew = fmaxf(mrow, mloc);
    const float corr = exp2f(mrow - mnew);
    float psum = 0.f;
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const float p = exp2f(s[jj] - mnew);
      psum += p;
      Ps[r * KS + jj * 4 + qd] = p;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    lrow = lrow * corr + psum;
    mrow = mnew;
    __syncwarp();
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] *= corr;
    for (int key = 0; key < BKV; ++key) {
      const float p = Ps[r * KS + key];
      const float* vr = Vs + key * KS + qd;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (qd + 4 * m < dh) acc[m] = fmaf(p, vr[4 * m], acc[m]);
    }
    __syncthreads();
  }
  if (q0 + r < L) {
    const float inv = 1.f / lrow;
    T* op = o + (size_t)qrow * d + h * dh;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int c = qd + 4 * m;
      if (c < dh) {
        if constexpr (sizeof(T) == 2) op[c] = __float2half_rn(acc[m] * inv);
        else op[c] = acc[m] * inv;
      }
    }
  }
}

}  // namespace

cudaError_t launch_attention_simt(const void* qk, const void* vt, Clips clips, void* o, int t_half, int rows_pad,
                                  int n_heads, int d_head, int t_max, cudaStream_t s) {
  if (d_head > 64 || d_head % 4) return cudaErrorInvalidValue;
  const float qscale = 1.4426950408889634f / sqrtf((float)d_head);
  dim3 grid((t_max + BQ - 1) / BQ, n_heads, clips.B);
  cudaError_t e;
  if (t_half) {
    e = cudaFuncSetAttribute(attn_simt_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    attn_simt_kernel<__half><<<grid, 256, SMEM, s>>>((const __half*)qk, (const __half*)vt, clips, (__half*)o,
                                                     rows_pad, n_heads, d_head, qscale);
  } else {
    e = cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    attn_simt_kernel<float><<<grid, 256, SMEM, s>>>((const float*)qk, (const float*)vt, clips, (float*)o, rows_pad,
                                                    n_heads, d_head, qscale);
  }
  return cudaGetLastError();
}

}  // namespace gam
