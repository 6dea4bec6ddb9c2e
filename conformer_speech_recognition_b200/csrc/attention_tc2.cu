// Masked multi-head self-attention on the sm_100a tensor cores, second form:
// 64-key blocks with the score tile double-buffered in TMEM and the softmax
// output P written back into TMEM, so the tensor core computes the next
// block's scores while the softmax works on the current one.
//
// softmax(Q K^T / sqrt(d_head) + mask) V per (clip, head); keys at or beyond
// the clip's valid length are masked ("GigaAM MLX port for Mac", "What is
// inside the model": masking is part of the reproduced path).
//
// CTA = 128 queries of one (clip, head), 192 threads, 2 CTAs per SM:
//   warp 0      TMA: the Q tile once, then 64-key K tiles and 64-key V^T tiles
//               into 3-stage rings (128-byte swizzle);
//   warp 1      TMEM (S0, S1: 64 columns each, O: d_head columns); one thread
//               issues S(0) and S(1) = Q K^T (M 128, N 64, K d_head), then per
//               block j, once P(j) is in TMEM: O += P(j) V(j) with A read from
//               TMEM (tcgen05.mma ... [a_tmem]), then S(j + 2) into the buffer
//               P(j) came from (issued after the P.V that reads it, and the
//               tensor core runs one thread's MMAs in order);
//   warps 2..5  softmax, one query row per thread (TMEM lane): the 64 scores
//               of a block are loaded once into registers; the exponent offset
//               only rises when a score exceeds it by 2^8 (then O, after the
//               previous P.V has finished, and the row sum are rescaled);
//               exp2 of the scaled scores, fp16 pairs stored over the scores
//               (32 TMEM columns), row sum in fp32; finally O / sum, read once
//               the MMA thread's closing commit (all MMAs done) has landed.
// Q, K come from the head-major buffer [2][H][rows][64] (head dim padded to
// 64) and V from V^T [H][64][rows]; clip starts are multiples of 8 rows, so
// every TMA x coordinate is 16-byte aligned.  All waits are bounded.
#include <cstdint>

#include "gemm_tc.cuh"
#include "tc_common.cuh"

namespace gam {

namespace {

using namespace tc;

constexpr int BQ = 128, BK2 = 64;
constexpr int KST = 3, VST = 3;           // K and V ring stages
constexpr int Q_BYTES = BQ * 64 * 2;      // 16 KB
constexpr int K_BYTES = BK2 * 64 * 2;     // 8 KB: 64 keys x 64 head dims
constexpr int V_BYTES = 64 * BK2 * 2;     // 8 KB: 64 head dims x 64 keys (one swizzle atom)
constexpr int SMEM_BYTES = Q_BYTES + KST * K_BYTES + VST * V_BYTES + 1024 + 256;
constexpr uint32_t TMEM_COLS = 256;       // S0: 0..63, S1: 64..127, O: 128..191
constexpr float kRescaleThreshold = 8.f;  // log2 units

struct AttnArgs {
  Clips clips;
  int n_heads, d_head, rows_pad;
  float scale_log2;  // log2(e) / sqrt(d_head)
  __half* out;       // [rows, d]
  int* status;
};

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16; A is M x 16 fp16 held as 8 TMEM
// columns of packed pairs (lane = row).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

// Packed fp32 pairs (sm_100 .f32x2 arithmetic): a 64-bit register holds two floats.
__device__ __forceinline__ uint64_t pack_f32x2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 unpack_f32x2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max of three floats in one instruction (sm_100); a NaN operand is ignored, as by fmaxf
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(192, 2)
attn_tc2_kernel(const __grid_constant__ CUtensorMap mQK, const __grid_constant__ CUtensorMap mVT, const AttnArgs p) {
  pdl_launch_dependents();
  pdl_wait();  // Q, K, V^T from the previous kernel are complete
  const int b = blockIdx.z, h = blockIdx.y;
  const int L = p.clips.L2(b), e0 = p.clips.e(b);
  const int q0 = blockIdx.x * BQ;
  if (q0 >= L) return;  // uniform for the whole CTA, before any barrier / TMEM use
  const int dh = p.d_head;
  const int nblk = (L + BK2 - 1) / BK2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;
  uint8_t* sK = sQ + Q_BYTES;            // [KST][K_BYTES]
  uint8_t* sV = sK + KST * K_BYTES;      // [VST][V_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VST * V_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;   // [KST]
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;  // [2] per score buffer
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tO = tmem + 128;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&mQK);
      prefetch_tmap(&mVT);
      const int qrow = h * p.rows_pad + e0 + q0;
      const int krow = (p.n_heads + h) * p.rows_pad + e0;
      // the 128-row Q tile as two 64-row boxes: rows 64 .. 127 land 8 KB further on, which
      // is exactly where one 128-row box would put them in the swizzled layout
      mbar_arrive_expect_tx(q_full, Q_BYTES);
      tma_load_2d(sQ, &mQK, q_full, 0, qrow);
      tma_load_2d(sQ + Q_BYTES / 2, &mQK, q_full, 0, qrow + 64);
      int nk = 0, nv = 0;
      for (int j = 0; j < nblk; ++j) {
        const int sk = j % KST, sv = j % VST;
        if (!mbar_wait(&k_empty[sk], ((j / KST) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[sk], K_BYTES);
        tma_load_2d(sK + sk * K_BYTES, &mQK, &k_full[sk], 0, krow + j * BK2);
        ++nk;
        if (!mbar_wait(&v_empty[sv], ((j / VST) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&v_full[sv], V_BYTES);
        tma_load_2d(sV + sv * V_BYTES, &mVT, &v_full[sv], e0 + j * BK2, h * 64);
        ++nv;
      }
      // copies in flight land before exit (bounded)
      mbar_settle(q_full, 0, abort_flag, kWaitLimitNs);
      for (int j = nk > KST ? nk - KST : 0; j < nk; ++j) mbar_settle(&k_full[j % KST], (j / KST) & 1, abort_flag, kWaitLimitNs);
      for (int j = nv > VST ? nv - VST : 0; j < nv; ++j) mbar_settle(&v_full[j % VST], (j / VST) & 1, abort_flag, kWaitLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16_f32(BQ, BK2);
      const uint32_t idesc_o = idesc_f16_f32(BQ, dh);
      const int ksteps_s = dh / 16;
      bool ok = mbar_wait(q_full, 0, abort_flag);
      const uint64_t dq = sdesc_k_sw128(smem_u32(sQ));
      // S(i) = Q K(i)^T into score buffer i % 2, then release the K stage
      auto issue_s = [&](int i) {
        const int sk = i % KST;
        if (!mbar_wait(&k_full[sk], (i / KST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dk = sdesc_k_sw128(smem_u32(sK + sk * K_BYTES));
        const uint32_t tS = tmem + (uint32_t)((i & 1) * BK2);
        for (int k = 0; k < ksteps_s; ++k) umma_f16(tS, dq + 2 * k, dk + 2 * k, idesc_s, k != 0 ? 1u : 0u);
        umma_commit(&s_full[i & 1]);
        umma_commit(&k_empty[sk]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nblk > 1) ok = issue_s(1);
      for (int j = 0; j < nblk && ok; ++j) {
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, abort_flag)) break;
        const int sv = j % VST;
        if (!mbar_wait(&v_full[sv], (j / VST) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t tP = tmem + (uint32_t)((j & 1) * BK2);  // P(j): 32 columns of fp16 pairs
        const uint64_t dv = sdesc_k_sw128(smem_u32(sV + sv * V_BYTES));
#pragma unroll
        for (int kk = 0; kk < BK2 / 16; ++kk)
          umma_f16_ts(tO, tP + (uint32_t)(kk * 8), dv + 2 * kk, idesc_o, (j | kk) != 0 ? 1u : 0u);
        umma_commit(o_full);
        umma_commit(&v_empty[sv]);
        if (j + 2 < nblk && !issue_s(j + 2)) break;  // after the P.V that reads this buffer
      }
      umma_commit(drain);
      mbar_settle(drain, 0, abort_flag, kWaitLimitNs);
    }
  } else {
    // softmax warps: query row r of the tile = TMEM lane
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_used = -INFINITY, l = 0.f;  // exponent offset in use (log2 units), row sum
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      const int buf = j & 1;
      const uint32_t tS = tmem + lane_off + (uint32_t)(buf * BK2);
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t u[2][32];
      tmem_ld32(tS, u[0]);
      tmem_ld32(tS + 32, u[1]);
      tmem_ld_wait();
      const int kvalid = L - j * BK2;  // keys [0, kvalid) of this block are valid
      // row maximum as 8 independent partial maxima (short dependency chains)
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = -INFINITY;
      if (kvalid >= BK2) {  // three-input maxima: 4 per 8 scores
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t = 8 * e;
          float m = fmax3(__uint_as_float(u[t >> 5][t & 31]), __uint_as_float(u[t >> 5][(t & 31) + 1]),
                          __uint_as_float(u[t >> 5][(t & 31) + 2]));
          m = fmax3(m, __uint_as_float(u[t >> 5][(t & 31) + 3]), __uint_as_float(u[t >> 5][(t & 31) + 4]));
          m = fmax3(m, __uint_as_float(u[t >> 5][(t & 31) + 5]), __uint_as_float(u[t >> 5][(t & 31) + 6]));
          pm[e] = fmaxf(m, __uint_as_float(u[t >> 5][(t & 31) + 7]));
        }
      } else {
#pragma unroll
        for (int t = 0; t < BK2; ++t)
          if (t < kvalid) pm[t & 7] = fmaxf(pm[t & 7], __uint_as_float(u[t >> 5][t & 31]));
      }
      float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      mx *= p.scale_log2;
      if (__any_sync(0xffffffffu, mx > m_used + kRescaleThreshold)) {
        // the previous P.V must have finished before O is rescaled (its phase j - 1)
        if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(o_full, (j - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool raise = mx > m_used + kRescaleThreshold;
        const float corr = raise ? fast_exp2(m_used - mx) : 1.f;  // 0 for the first block
        if (j > 0) {
#pragma unroll 1
          for (int c = 0; c < dh; c += 32) {  // dh in {48, 64}: columns [c, c+32) (the tail is unused)
            uint32_t o[32];
            tmem_ld32(tO + lane_off + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * corr);
            tmem_st32(tO + lane_off + c, o);
          }
          tmem_st_wait();
        }
        if (raise) {
          l *= corr;
          m_used = mx;
        }
      }
      // exponentials, row sum, fp16 pairs of P over the scores (32 columns).  Scores go
      // in pairs through packed fp32 ops (one fma.rn.f32x2 for both exponent arguments,
      // one add.rn.f32x2 into 4 partial pair sums); each lane of a pair is still one
      // fp32 fma / add.
      const uint64_t sc2 = pack_f32x2(p.scale_log2, p.scale_log2), nm2 = pack_f32x2(-m_used, -m_used);
      uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pw[32];
      if (kvalid >= BK2) {
#pragma unroll
        for (int t = 0; t < BK2; t += 2) {
          const float2 z = unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(u[t >> 5][t & 31]),
                                                             __uint_as_float(u[t >> 5][(t & 31) + 1])),
                                                  sc2, nm2));
          const float a0 = fast_exp2(z.x), a1 = fast_exp2(z.y);
          ps2[(t >> 1) & 3] = add_f32x2(ps2[(t >> 1) & 3], pack_f32x2(a0, a1));
          __half2 hv = __floats2half2_rn(a0, a1);
          pw[t >> 1] = *reinterpret_cast<uint32_t*>(&hv);
        }
      } else {
#pragma unroll
        for (int t = 0; t < BK2; t += 2) {
          const float2 z = unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(u[t >> 5][t & 31]),
                                                             __uint_as_float(u[t >> 5][(t & 31) + 1])),
                                                  sc2, nm2));
          const float a0 = t < kvalid ? fast_exp2(z.x) : 0.f, a1 = t + 1 < kvalid ? fast_exp2(z.y) : 0.f;
          ps2[(t >> 1) & 3] = add_f32x2(ps2[(t >> 1) & 3], pack_f32x2(a0, a1));
          __half2 hv = __floats2half2_rn(a0, a1);
          pw[t >> 1] = *reinterpret_cast<uint32_t*>(&hv);
        }
      }
      {
        const float2 q = unpack_f32x2(add_f32x2(add_f32x2(ps2[0], ps2[1]), add_f32x2(ps2[2], ps2[3])));
        l += q.x + q.y;
      }
      tmem_st32(tS, pw);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[buf]);
    }
    // epilogue: O / l once every MMA has finished.  Here P.V(nblk - 2) may still be
    // in flight as well as P.V(nblk - 1) (S(nblk - 1) was issued before it), so a
    // parity wait on o_full could see the phase of P.V(nblk - 3) and pass early;
    // `drain` completes once, after the MMA thread's last commit.
    if (ok && !__all_sync(0xffffffffu, mbar_wait(drain, 0, abort_flag))) ok = false;
    tc_fence_after();
    uint32_t o0[32], o1[32];
    tmem_ld32(tO + lane_off, o0);
    tmem_ld32(tO + lane_off + 32, o1);
    tmem_ld_wait();
    if (ok && q0 + r < L) {
      const float inv = 1.f / l;
      __half* o = p.out + (size_t)(e0 + q0 + r) * (p.n_heads * dh) + h * dh;
#pragma unroll
      for (int c = 0; c < 64; c += 8) {
        if (c < dh) {
          uint4 w;
          uint32_t* pv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = c + 2 * e;
            const float a0 = __uint_as_float(k0 < 32 ? o0[k0] : o1[k0 - 32]);
            const float a1 = __uint_as_float(k0 + 1 < 32 ? o0[k0 + 1] : o1[k0 + 1 - 32]);
            __half2 hv = __floats2half2_rn(a0 * inv, a1 * inv);
            pv[e] = *reinterpret_cast<uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(o + c) = w;
        }
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

// fp16 rows of `inner` elements, 128-byte swizzle.
cudaError_t map2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer) {
  return tma_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ptr, inner, outer, inner * 2, box_inner, box_outer,
                    CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_attention_tc2(TcGemmCache* cache, const void* qk, const void* vt, Clips clips, void* o,
                                 int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s) {
  if ((d_head != 48 && d_head != 64) || rows_pad % 8) return cudaErrorInvalidValue;
  CUtensorMap mQK, mVT;
  // one 64-row box for K tiles and both halves of a Q tile
  cudaError_t e = map2d(&mQK, qk, 64, (uint64_t)2 * n_heads * rows_pad, 64, BK2);
  if (e == cudaSuccess) e = map2d(&mVT, vt, rows_pad, (uint64_t)n_heads * 64, BK2, 64);
  if (e != cudaSuccess) return e;
  AttnArgs a;
  a.clips = clips;
  a.n_heads = n_heads;
  a.d_head = d_head;
  a.rows_pad = rows_pad;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d_head);
  a.out = reinterpret_cast<__half*>(o);
  a.status = cache->status;
  e = cudaFuncSetAttribute(attn_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((t_max + BQ - 1) / BQ, n_heads, clips.B);
  return launch_pdl(attn_tc2_kernel, grid, 192, SMEM_BYTES, s, mQK, mVT, a);
}

}  // namespace gam
