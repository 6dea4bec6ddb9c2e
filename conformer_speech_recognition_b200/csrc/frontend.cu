// Log-mel frontend of the fp32 build mode, on CUDA cores ("GigaAM v3 MLX",
// "Frontend configuration"; "GigaAM v3 RNNT -- MLX (Apple Silicon)", "Notes for
// other runtimes").  The fp16 / INT8 product modes use the tensor-core frontend
// of frontend_tc.cu.
//
// Per frame f of clip i: x = audio[i, 160 f .. 160 f + 319] (center=false).
// The stored Hann window is folded into a real-DFT basis built at context
// creation: basis[n][k] = w[n] cos(2 pi k n / 320) for k = 0..160 and
// basis[n][160 + k] = w[n] sin(2 pi k n / 320) for k = 1..159, so one fp32
// GEMM row gives the real and imaginary parts of all 161 bins.  Power 2,
// then the stored filterbank [161, 64] (no normalisation), then
// log(clip(., 1e-9, 1e9)).
//
// One CTA handles 32 frames: the frames are staged in shared memory, the
// basis is streamed through shared memory in chunks of 32 samples, the power
// spectrum replaces the frames in shared memory and the filterbank replaces
// the basis.  Output rows are either the packed mel rows of the encoder
// (segment layout, fp16 or fp32, zero rows between clips) or the padded
// [B, F_max, 64] fp32 output of gam_logmel.
#include "common.cuh"

namespace gam {
namespace {

constexpr int FT = 32;      // frames per CTA
constexpr int NFFT = 320;   // n_fft = window
constexpr int HOP = 160;
constexpr int NBIN = 161;   // n_fft / 2 + 1
constexpr int NMEL = 64;
constexpr int NCH = 32;     // samples per basis chunk
constexpr int FRAME_FLOATS = FT * NFFT;                  // 10240
constexpr int BASIS_FLOATS = NBIN * NMEL;                // 10304 >= NCH * NFFT (10240)
constexpr size_t SMEM_BYTES = (FRAME_FLOATS + BASIS_FLOATS) * sizeof(float);

__global__ void __launch_bounds__(256)
frontend_kernel(const float* __restrict__ audio, int64_t stride, Clips clips, int rows, int packed, int f_max,
                const float* __restrict__ basis, const float* __restrict__ fb, void* __restrict__ out,
                int out_half) {
  extern __shared__ __align__(16) float sm[];
  float* fr = sm;                  // [FT][NFFT] frames, later [FT][NBIN] power
  float* bs = sm + FRAME_FLOATS;   // [NCH][NFFT] basis chunk, later [NBIN][NMEL] filterbank
  __shared__ int s_clip[FT], s_frame[FT];

  const int tid = threadIdx.x;
  const int row0 = blockIdx.x * FT;
  if (tid < FT) {
    const int r = row0 + tid;
    int ci = -1, f = -1;
    if (r < rows) {
      if (packed) {
        ci = clips.find(r, 4, 6);
        f = r - (4 * clips.e(ci) + 6);
      } else {
        ci = r / f_max;
        f = r - ci * f_max;
      }
      if (f < 0 || f >= clips.F(ci)) ci = -1;
    }
    s_clip[tid] = ci;
    s_frame[tid] = f;
  }
  __syncthreads();

  // stage frames (zeros for rows outside every clip)
  for (int idx = tid; idx < FRAME_FLOATS; idx += 256) {
    const int j = idx / NFFT, n = idx - j * NFFT;
    const int ci = s_clip[j];
    fr[idx] = ci >= 0 ? __ldg(audio + (int64_t)ci * stride + (int64_t)s_frame[j] * HOP + n) : 0.f;
  }

  // DFT: warp w owns frames 4w .. 4w+3; lane owns bins lane + 32 q (q < 6, bin < 161)
  const int warp = tid >> 5, lane = tid & 31;
  float re[4][6], im[4][6];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int q = 0; q < 6; ++q) re[a][q] = im[a][q] = 0.f;

  for (int n0 = 0; n0 < NFFT; n0 += NCH) {
    __syncthreads();
    for (int idx = tid; idx < NCH * NFFT; idx += 256) bs[idx] = __ldg(basis + (size_t)n0 * NFFT + idx);
    __syncthreads();
    // blocked summation: partial sums over 32 samples, then added to the totals
    float pre[4][6], pim[4][6];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int q = 0; q < 6; ++q) pre[a][q] = pim[a][q] = 0.f;
#pragma unroll 4
    for (int nn = 0; nn < NCH; ++nn) {
      float xv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) xv[a] = fr[(warp * 4 + a) * NFFT + n0 + nn];
      const float* brow = bs + nn * NFFT;
#pragma unroll
      for (int q = 0; q < 6; ++q) {
        const int k = lane + 32 * q;
        if (k < NBIN) {
          const float c = brow[k];
          const float s = (k >= 1 && k <= 159) ? brow[160 + k] : 0.f;
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            pre[a][q] = fmaf(xv[a], c, pre[a][q]);
            pim[a][q] = fmaf(xv[a], s, pim[a][q]);
          }
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int q = 0; q < 6; ++q) {
        re[a][q] += pre[a][q];
        im[a][q] += pim[a][q];
      }
  }
  __syncthreads();
  // power spectrum into fr as [FT][NBIN]
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int q = 0; q < 6; ++q) {
      const int k = lane + 32 * q;
      if (k < NBIN) fr[(warp * 4 + a) * NBIN + k] = re[a][q] * re[a][q] + im[a][q] * im[a][q];
    }
  for (int idx = tid; idx < NBIN * NMEL; idx += 256) bs[idx] = __ldg(fb + idx);
  __syncthreads();

  // mel + log: thread owns mel m = tid % 64 for frames tid/64 + 4 j
  const int m = tid & 63;
#pragma unroll
  for (int j = 0; j < FT / 4; ++j) {
    const int a = (tid >> 6) + 4 * j;
    const float* P = fr + a * NBIN;
    float acc = 0.f;
    for (int k = 0; k < NBIN; ++k) acc = fmaf(P[k], bs[k * NMEL + m], acc);
    const int r = row0 + a;
    if (r >= rows) continue;
    const float v = s_clip[a] >= 0 ? logf(fminf(fmaxf(acc, 1e-9f), 1e9f)) : 0.f;
    if (out_half) reinterpret_cast<__half*>(out)[(size_t)r * NMEL + m] = __float2half_rn(v);
    else reinterpret_cast<float*>(out)[(size_t)r * NMEL + m] = v;
  }
}

}  // namespace

cudaError_t launch_frontend(const float* audio, int64_t audio_stride, Clips clips, int rows, int packed, int f_max,
                            const float* basis, const float* fb, void* out, int out_half, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(frontend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (rows <= 0) return cudaSuccess;
  frontend_kernel<<<(rows + FT - 1) / FT, 256, SMEM_BYTES, s>>>(audio, audio_stride, clips, rows, packed, f_max,
                                                                 basis, fb, out, out_half);
  return cudaGetLastError();
}

}  // namespace gam
