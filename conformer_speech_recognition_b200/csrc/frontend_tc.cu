// Log-mel frontend of the fp16 / INT8 product modes on the sm_100a tensor cores,
// at fp32 accuracy ("GigaAM v3 MLX", "Frontend configuration": window 320,
// hop 160, n_fft 320, center false, power 2, 64 HTK mel bins without
// normalisation; "GigaAM v3 RNNT -- MLX (Apple Silicon)", "Notes for other
// runtimes": the stored window and filterbank, log(clip(x, 1e-9, 1e9)); the
// pages compare their log-mel with an fp32 reference to 3e-5 ("GigaAM on MLX:
// the transcripts matched, but the model was broken", "Trap 3")).
//
// Two kernels:
//  * audio_split_kernel writes every clip's samples in the packed mel-row
//    layout of common.cuh as rows of one hop (160 samples): packed row
//    4 e_i + 6 + g holds samples [160 g, 160 g + 160) of clip i for
//    g = 0 .. F_i, so frame f of the clip is the pair of rows (f, f + 1) and
//    the DFT's A operand is a plain 2D view with no frame buffer.  Each sample
//    x is stored as x_hi = tf32(x) and x_lo = tf32(x - x_hi); rows outside
//    every clip are zero.
//  * dft_mel_tf32_kernel: one CTA per 128 frames.  The windowed real DFT
//    (basis rows [cos 64 bins | sin 64 bins] per 128 columns, bins 0 .. 191,
//    the Hann window folded in) runs on tcgen05 with kind::tf32 as three
//    products, A_hi B_hi + A_lo B_hi + A_hi B_lo (the dropped A_lo B_lo term
//    and the tf32 rounding of the parts leave a relative error near 2^-21 per
//    product), accumulated in fp32 in TMEM: 3 accumulators of 128 x 128.  The
//    epilogue squares and adds the cos / sin columns into the power spectrum
//    (161 bins, one shared-memory row per frame), applies the filterbank over
//    each mel bin's nonzero rows and writes log(clip(mel, 1e-9, 1e9)).
//
// Warp roles (192 threads): warp 0 issues the TMA loads (A: the hi and lo rows
// of the 128 frames, 32 samples per stage; B: the hi and lo basis tiles of one
// 128-column block per stage), warp 1 allocates TMEM and one thread issues the
// MMAs, warps 2..5 run the epilogue (warp w reads TMEM lanes 32 (w % 4) ..).
// Every wait is bounded (tc_common.cuh).
#include <cstdint>

#include "gemm_tc.cuh"
#include "tc_common.cuh"

namespace gam {
namespace {

using namespace tc;

constexpr int FBM = 128;          // frames (packed mel rows) per CTA
constexpr int HOPN = 160;         // samples per packed row
constexpr int KCH = 32;           // samples per stage: 128-byte rows of fp32
constexpr int NKC = 320 / KCH;    // 10 stages cover a frame (two packed rows)
constexpr int NJ = 3;             // 128-column basis blocks (bins 0 .. 191)
constexpr int NBIN = 161, NMEL = 64;
constexpr int OP_TILE = 128 * KCH * 4;          // one 128 x 32 fp32 operand tile (16 KB)
constexpr int SA = 2, SB = 4;                   // A and B ring depths
constexpr int A_STAGE = 2 * OP_TILE;            // hi + lo
constexpr int B_STAGE = 2 * OP_TILE;
constexpr int RING = SA * A_STAGE + SB * B_STAGE;  // 192 KB
constexpr int PROW = NBIN;  // floats per power row: odd, so a warp's rows fall in distinct banks
constexpr int FB_OFF = (FBM * PROW * 4 + 15) / 16 * 16;  // filterbank copy after the power rows
static_assert(FB_OFF + NBIN * NMEL * 4 <= RING, "the power rows and the filterbank reuse the operand ring");
constexpr size_t SMEM_BYTES = RING + 1024 + 256;
constexpr uint32_t TMEM_COLS = 512;  // 3 x 128 accumulator columns, rounded to a power of two

// Instruction descriptor of kind::tf32: TF32 A and B (both K-major), fp32
// accumulator, M x N tile.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4)                      // accumulator format F32
         | (2u << 7) | (2u << 10)       // A, B format TF32
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::tf32 (K = 8 per instruction).
__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

// Round to the nearest tf32 value (ties away from zero), returned as fp32.
__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <bool VEC>
__global__ void __launch_bounds__(256)
audio_split_kernel(const float* __restrict__ audio, int64_t stride, Clips clips, int rows, float* __restrict__ hi,
                   float* __restrict__ lo) {
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int ci = clips.find(r, 4, 6);
  const int g = r - (4 * clips.e(ci) + 6);
  // F frames need F + 1 rows; row F ends at sample 160 F + 159 < N
  const bool valid = g >= 0 && g <= clips.F(ci);
  const float* src = audio + (int64_t)ci * stride + (int64_t)g * HOPN;
  for (int c = lane * 4; c < HOPN; c += 128) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid) {
      if (VEC) v = __ldg(reinterpret_cast<const float4*>(src + c));
      else v = make_float4(__ldg(src + c), __ldg(src + c + 1), __ldg(src + c + 2), __ldg(src + c + 3));
    }
    const float4 h = make_float4(to_tf32(v.x), to_tf32(v.y), to_tf32(v.z), to_tf32(v.w));
    const float4 l = make_float4(to_tf32(v.x - h.x), to_tf32(v.y - h.y), to_tf32(v.z - h.z), to_tf32(v.w - h.w));
    *reinterpret_cast<float4*>(hi + (size_t)r * HOPN + c) = h;
    *reinterpret_cast<float4*>(lo + (size_t)r * HOPN + c) = l;
  }
}

struct DftArgs {
  Clips clips;
  int rows;             // packed mel rows (frames) to compute
  int mode;             // 0: fp16 packed rows, zero outside clips; 1: fp32 [B, f_max, 64], valid rows only
  int f_max;
  void* out;
  const float* fb;      // [161][64] filterbank
  const int2* fb_range; // per mel bin: first and last nonzero filterbank row
  int* status;
};

__global__ void __launch_bounds__(192, 1)
dft_mel_tf32_kernel(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
                    const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
                    const DftArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;                 // [SA][hi | lo] frame tiles
  uint8_t* sB = base + SA * A_STAGE;  // [SB][hi | lo] basis tiles
  uint64_t* a_full = reinterpret_cast<uint64_t*>(base + RING);
  uint64_t* a_empty = a_full + SA;
  uint64_t* b_full = a_empty + SA;
  uint64_t* b_empty = b_full + SB;
  uint64_t* acc_full = b_empty + SB;
  uint64_t* drain = acc_full + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mAh);
    prefetch_tmap(&mAl);
    prefetch_tmap(&mBh);
    prefetch_tmap(&mBl);
  }
  if (warp == 1) tmem_alloc(tslot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_launch_dependents();
  pdl_wait();  // the split audio from the previous kernel is complete
  const int m0 = blockIdx.x * FBM;

  if (warp == 0) {
    if (lane == 0) {
      int na = 0, nb = 0;  // stages issued
      bool ok = true;
      for (int kc = 0; kc < NKC && ok; ++kc) {
        const int sa = kc % SA;
        if (!mbar_wait(&a_empty[sa], ((kc / SA) & 1) ^ 1, abort_flag)) break;
        // samples 32 (kc % 5) .. of packed row m0 + kc / 5 (frame = rows f, f + 1)
        const int x = (kc % 5) * KCH, y = m0 + kc / 5;
        mbar_arrive_expect_tx(&a_full[sa], A_STAGE);
        tma_load_2d(sA + sa * A_STAGE, &mAh, &a_full[sa], x, y);
        tma_load_2d(sA + sa * A_STAGE + OP_TILE, &mAl, &a_full[sa], x, y);
        ++na;
        for (int j = 0; j < NJ; ++j) {
          const int sb = nb % SB;
          if (!mbar_wait(&b_empty[sb], ((nb / SB) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&b_full[sb], B_STAGE);
          tma_load_2d(sB + sb * B_STAGE, &mBh, &b_full[sb], kc * KCH, j * 128);
          tma_load_2d(sB + sb * B_STAGE + OP_TILE, &mBl, &b_full[sb], kc * KCH, j * 128);
          ++nb;
        }
      }
      // every issued copy lands before the CTA can exit (bounded)
      for (int i = na > SA ? na - SA : 0; i < na; ++i) mbar_settle(&a_full[i % SA], (i / SA) & 1, abort_flag, kWaitLimitNs);
      for (int i = nb > SB ? nb - SB : 0; i < nb; ++i) mbar_settle(&b_full[i % SB], (i / SB) & 1, abort_flag, kWaitLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32_f32(FBM, 128);
      int nb = 0;
      bool ok = true;
      for (int kc = 0; kc < NKC && ok; ++kc) {
        const int sa = kc % SA;
        if (!mbar_wait(&a_full[sa], (kc / SA) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dah = sdesc_k_sw128(smem_u32(sA + sa * A_STAGE));
        const uint64_t dal = sdesc_k_sw128(smem_u32(sA + sa * A_STAGE + OP_TILE));
        for (int j = 0; j < NJ; ++j) {
          const int sb = nb % SB;
          if (!mbar_wait(&b_full[sb], (nb / SB) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dbh = sdesc_k_sw128(smem_u32(sB + sb * B_STAGE));
          const uint64_t dbl = sdesc_k_sw128(smem_u32(sB + sb * B_STAGE + OP_TILE));
          const uint32_t d = tmem + (uint32_t)(j * 128);
#pragma unroll
          for (int k = 0; k < KCH / 8; ++k) {  // 8 samples (32 bytes) per instruction
            umma_tf32(d, dah + 2 * k, dbh + 2 * k, idesc, (kc | k) != 0 ? 1u : 0u);
            umma_tf32(d, dal + 2 * k, dbh + 2 * k, idesc, 1u);
            umma_tf32(d, dah + 2 * k, dbl + 2 * k, idesc, 1u);
          }
          umma_commit(&b_empty[sb]);
          ++nb;
        }
        if (ok) umma_commit(&a_empty[sa]);
      }
      if (ok) umma_commit(acc_full);
      umma_commit(drain);  // every MMA issued above completes before TMEM is freed (bounded)
      mbar_settle(drain, 0, abort_flag, kWaitLimitNs);
    }
  } else {
    // epilogue: frame (row) r_local = TMEM lane
    const int q = warp & 3;
    const int rl = q * 32 + lane, r = m0 + rl;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag));
    tc_fence_after();
    // the operand ring is idle now (every MMA has completed): power rows and a copy
    // of the filterbank go there; the four epilogue warps share the copy, and all of
    // them pass the barrier below whether or not their wait succeeded
    float* P = reinterpret_cast<float*>(base) + rl * PROW;
    float* fbs = reinterpret_cast<float*>(base + FB_OFF);
    if (ok)
      for (int i = rl; i < NBIN * NMEL / 4; i += FBM)
        reinterpret_cast<float4*>(fbs)[i] = __ldg(reinterpret_cast<const float4*>(p.fb) + i);
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the filterbank copy is complete
    if (ok) {
#pragma unroll 1
      for (int j = 0; j < NJ; ++j) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t cr[32], si[32];
          tmem_ld32(tmem + lane_off + (uint32_t)(j * 128 + h * 32), cr);
          tmem_ld32(tmem + lane_off + (uint32_t)(j * 128 + 64 + h * 32), si);
          tmem_ld_wait();
          const int k0 = j * 64 + h * 32;
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float a = __uint_as_float(cr[t]), b = __uint_as_float(si[t]);
            if (k0 + t < NBIN) P[k0 + t] = fmaf(a, a, b * b);
          }
        }
      }
      int ci = -1, f = -1;
      if (r < p.rows) {
        ci = p.clips.find(r, 4, 6);
        f = r - (4 * p.clips.e(ci) + 6);
        if (f < 0 || f >= p.clips.F(ci)) ci = -1;
      }
      float v[NMEL];
#pragma unroll
      for (int m = 0; m < NMEL; ++m) {
        const int2 kr = __ldg(p.fb_range + m);
        float acc = 0.f;
#pragma unroll 4
        for (int k = kr.x; k <= kr.y; ++k) acc = fmaf(P[k], fbs[k * NMEL + m], acc);
        v[m] = ci >= 0 ? logf(fminf(fmaxf(acc, 1e-9f), 1e9f)) : 0.f;
      }
      if (p.mode == 0) {
        if (r < p.rows) {
          uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.out) + (size_t)r * NMEL);
#pragma unroll
          for (int c = 0; c < NMEL / 8; ++c) {
            uint4 w;
            uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __half2 hv = __floats2half2_rn(v[8 * c + 2 * e], v[8 * c + 2 * e + 1]);
              pw[e] = *reinterpret_cast<uint32_t*>(&hv);
            }
            o[c] = w;
          }
        }
      } else if (ci >= 0) {
        float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) +
                                              ((size_t)ci * p.f_max + f) * NMEL);
#pragma unroll
        for (int c = 0; c < NMEL / 4; ++c) o[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// 2D fp32 map, rows of `inner` floats, box 32 x 128 (128-byte swizzle), zero fill.
cudaError_t map_f32(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer) {
  return tma_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ptr, inner, outer, inner * 4, KCH, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_audio_split(const float* audio, int64_t audio_stride, Clips clips, int rows, float* hi, float* lo,
                               cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const bool vec = audio_stride % 4 == 0 && (reinterpret_cast<uintptr_t>(audio) & 15) == 0;
  if (vec) return launch_pdl(audio_split_kernel<true>, (rows + 7) / 8, 256, 0, s, audio, audio_stride, clips, rows, hi, lo);
  return launch_pdl(audio_split_kernel<false>, (rows + 7) / 8, 256, 0, s, audio, audio_stride, clips, rows, hi, lo);
}

cudaError_t launch_dft_mel(TcGemmCache* cache, const float* hi, const float* lo, int split_rows, const float* basis_hi,
                           const float* basis_lo, const float* fb, const int* fb_range, Clips clips, int rows,
                           int mode, int f_max, void* out, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (split_rows < rows + 1) return cudaErrorInvalidValue;  // frame f reads rows f and f + 1
  CUtensorMap mAh, mAl, mBh, mBl;
  cudaError_t e = map_f32(&mAh, hi, HOPN, (uint64_t)split_rows);
  if (e == cudaSuccess) e = map_f32(&mAl, lo, HOPN, (uint64_t)split_rows);
  if (e == cudaSuccess) e = map_f32(&mBh, basis_hi, 320, NJ * 128);
  if (e == cudaSuccess) e = map_f32(&mBl, basis_lo, 320, NJ * 128);
  if (e != cudaSuccess) return e;
  DftArgs a;
  a.clips = clips;
  a.rows = rows;
  a.mode = mode;
  a.f_max = f_max;
  a.out = out;
  a.fb = fb;
  a.fb_range = reinterpret_cast<const int2*>(fb_range);
  a.status = cache->status;
  e = cudaFuncSetAttribute(dft_mel_tf32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(dft_mel_tf32_kernel, (rows + FBM - 1) / FBM, 192, SMEM_BYTES, s, mAh, mAl, mBh, mBl, a);
}

}  // namespace gam
