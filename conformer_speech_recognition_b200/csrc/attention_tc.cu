// Masked multi-head self-attention on the sm_100a tensor cores (fp16 in,
// fp32 softmax and accumulation), flash style: one pass over the keys with an
// online softmax, never materialising the T' x T' score matrix in memory.
//
// softmax(Q K^T / sqrt(d_head) + mask) V per (clip, head); keys at or beyond
// the clip's valid length are masked ("GigaAM MLX port for Mac", "What is
// inside the model": masking is part of the reproduced path).
//
// CTA = 128 queries of one (clip, head), 192 threads:
//   warp 0      TMA: Q tile once, then K tiles of 128 keys into a 2-stage
//               ring and V^T tiles into a single buffer (128-byte swizzle);
//   warp 1      TMEM allocation; one thread issues S = Q K^T (M=128, N=128,
//               K=d_head) into TMEM and, once the softmax has turned S into
//               P, first the next block's S and then O_blk = P V (M=128,
//               N=d_head, K=128) with P read from shared memory;
//   warps 2..5  softmax, one query row per thread (TMEM lane): pass 1 takes
//               the row max of S (overlapping the previous block's P.V),
//               pass 2 writes exp2 / fp16 P into the swizzled shared-memory
//               operand layout.  O accumulates in TMEM across key blocks; it
//               is rescaled in place (tcgen05.ld / st) only when the running
//               max rises by more than 2^8, and divided by the row sum at the
//               end.
// Q, K come from the head-major buffer [2][H][rows][64] (head dim padded to
// 64) and V from V^T [H][64][rows]; clip starts are multiples of 8 rows so
// every TMA x coordinate is 16-byte aligned.  All waits are bounded.
#include <cstdint>

#include "gemm_tc.cuh"
#include "tc_common.cuh"

namespace gam {

namespace {

using namespace tc;

constexpr int BQ = 128, BKV = 128;
constexpr int Q_BYTES = BQ * 64 * 2;      // 16 KB
constexpr int K_BYTES = BKV * 64 * 2;     // 16 KB
constexpr int V_BYTES = 64 * BKV * 2;     // 16 KB (two 64-key swizzle atoms of 64 rows)
constexpr int P_BYTES = BQ * BKV * 2;     // 32 KB (two 64-key swizzle atoms of 128 rows)
constexpr int SMEM_BYTES = Q_BYTES + 2 * K_BYTES + V_BYTES + P_BYTES + 1024 + 256;  // 2 CTAs per SM
constexpr uint32_t TMEM_COLS = 256;       // S: columns 0..127, O: 128..191

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

// 2^x with the hardware approximation (ex2.approx, relative error ~2^-22),
// plenty for softmax weights that are rounded to fp16 afterwards.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Lazy rescaling threshold (log2 units): the running max used for the
// exponentials is only raised when a new score exceeds it by more than this,
// so P <= 2^8 stays well inside fp16 and O in TMEM is rarely rescaled.
constexpr float kRescaleThreshold = 8.f;

__global__ void __launch_bounds__(192, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap mQK, const __grid_constant__ CUtensorMap mVT, const AttnArgs p) {
  pdl_launch_dependents();
  pdl_wait();  // Q, K, V^T from the previous kernel are complete
  const int b = blockIdx.z, h = blockIdx.y;
  const int L = p.clips.L2(b), e0 = p.clips.e(b);
  const int q0 = blockIdx.x * BQ;
  if (q0 >= L) return;  // uniform for the whole CTA, before any barrier / TMEM use
  const int dh = p.d_head;
  const int nblk = (L + BKV - 1) / BKV;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = base;
  uint8_t* sK = sQ + Q_BYTES;             // [2][K_BYTES]
  uint8_t* sV = sK + 2 * K_BYTES;         // V_BYTES
  uint8_t* sP = sV + V_BYTES;             // P_BYTES
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + P_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 6;
  uint64_t* s_full = bars + 7;
  uint64_t* p_full = bars + 8;
  uint64_t* o_full = bars + 9;
  uint64_t* drain = bars + 11;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
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
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&mQK);
      prefetch_tmap(&mVT);
      const int qrow = h * p.rows_pad + e0 + q0;
      const int krow = (p.n_heads + h) * p.rows_pad + e0;
      mbar_arrive_expect_tx(q_full, Q_BYTES);
      tma_load_2d(sQ, &mQK, q_full, 0, qrow);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&k_empty[s], ((j >> 1) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[s], K_BYTES);
        tma_load_2d(sK + s * K_BYTES, &mQK, &k_full[s], 0, krow + j * BKV);
        ++k_issued;
        if (!mbar_wait(v_empty, (j & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(v_full, V_BYTES);
        tma_load_2d(sV, &mVT, v_full, e0 + j * BKV, h * 64);
        tma_load_2d(sV + V_BYTES / 2, &mVT, v_full, e0 + j * BKV + 64, h * 64);
        ++v_issued;
      }
      // copies in flight land before exit (bounded)
      auto settle = [&](uint64_t* bar, uint32_t parity) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar, parity))
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            break;
          }
      };
      settle(q_full, 0);
      for (int j = k_issued > 2 ? k_issued - 2 : 0; j < k_issued; ++j) settle(&k_full[j & 1], (j >> 1) & 1);
      if (v_issued > 0) settle(v_full, (v_issued - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16_f32(BQ, BKV);
      const uint32_t idesc_o = idesc_f16_f32(BQ, dh);
      const int ksteps_s = dh / 16;
      bool ok = mbar_wait(q_full, 0, abort_flag);
      const uint64_t dq = sdesc_k_sw128(smem_u32(sQ));
      // S(j) = Q K(j)^T into TMEM, then release the K stage
      auto issue_s = [&](int j) {
        const int s = j & 1;
        if (!mbar_wait(&k_full[s], (j >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dk = sdesc_k_sw128(smem_u32(sK + s * K_BYTES));
        for (int k = 0; k < ksteps_s; ++k) umma_f16(tS, dq + 2 * k, dk + 2 * k, idesc_s, k != 0 ? 1u : 0u);
        umma_commit(s_full);
        umma_commit(&k_empty[s]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nblk && ok; ++j) {
        // once the softmax has consumed S(j) (P(j) written), S(j+1) goes first so the
        // next softmax pass starts while P(j).V(j) runs
        if (!mbar_wait(p_full, j & 1, abort_flag)) break;
        if (j + 1 < nblk && !issue_s(j + 1)) break;
        if (!mbar_wait(v_full, j & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t pbase = smem_u32(sP), vbase = smem_u32(sV);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t da = sdesc_k_sw128(pbase + (kk >> 2) * (P_BYTES / 2)) + 2 * (kk & 3);
          const uint64_t db = sdesc_k_sw128(vbase + (kk >> 2) * (V_BYTES / 2)) + 2 * (kk & 3);
          umma_f16(tO, da, db, idesc_o, (j | kk) != 0 ? 1u : 0u);  // O accumulates across key blocks
        }
        umma_commit(o_full);
        umma_commit(v_empty);
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0))
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          *abort_flag = 1;
          break;
        }
    }
  } else {
    // softmax warps: query row r of the tile = TMEM lane
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float m_used = -INFINITY, l = 0.f;  // exponent offset in use (log2 units), row sum
    uint8_t* prow = sP + r * 128;        // row r inside each 64-key atom
    const int sw = r & 7;
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      // wait outcomes are made warp-uniform: the tcgen05 loads below are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int kvalid = L - j * BKV;  // keys [0, kvalid) of this block are valid
      // pass 1: row max of the raw scores (scale > 0 commutes with max), 64 columns per TMEM wait
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < BKV; c += 64) {
        uint32_t u[2][32];
        tmem_ld32(tS + lane_off + c, u[0]);
        tmem_ld32(tS + lane_off + c + 32, u[1]);
        tmem_ld_wait();
        if (c + 64 <= kvalid) {
#pragma unroll
          for (int t = 0; t < 64; ++t) mx = fmaxf(mx, __uint_as_float(u[t >> 5][t & 31]));
        } else {
#pragma unroll
          for (int t = 0; t < 64; ++t)
            if (c + t < kvalid) mx = fmaxf(mx, __uint_as_float(u[t >> 5][t & 31]));
        }
      }
      mx *= p.scale_log2;
      // P and O of the previous block: P.V(j-1) must have finished reading P and writing O
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(o_full, (j - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (mx > m_used + kRescaleThreshold) {
        const float corr = fast_exp2(m_used - mx);  // 0 for the first block
        if (j > 0) {
#pragma unroll 1
          for (int c = 0; c < dh; c += 32) {  // dh in {48, 64}: rescale columns [c, c+32) (the tail is unused)
            uint32_t o[32];
            tmem_ld32(tO + lane_off + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * corr);
            tmem_st32(tO + lane_off + c, o);
          }
          tmem_st_wait();
        }
        l *= corr;
        m_used = mx;
      }
      // pass 2: exponentials, row sum, fp16 P into the swizzled operand layout; one
      // 64-key swizzle atom (64 columns) per TMEM wait
      float sum = 0.f;
#pragma unroll 1
      for (int c = 0; c < BKV; c += 64) {
        uint32_t u[2][32];
        tmem_ld32(tS + lane_off + c, u[0]);
        tmem_ld32(tS + lane_off + c + 32, u[1]);
        tmem_ld_wait();
        float pv[64];
        if (c + 64 <= kvalid) {
#pragma unroll
          for (int t = 0; t < 64; ++t)
            pv[t] = fast_exp2(fmaf(__uint_as_float(u[t >> 5][t & 31]), p.scale_log2, -m_used));
        } else {
#pragma unroll
          for (int t = 0; t < 64; ++t)
            pv[t] = (c + t < kvalid) ? fast_exp2(fmaf(__uint_as_float(u[t >> 5][t & 31]), p.scale_log2, -m_used))
                                     : 0.f;
        }
#pragma unroll
        for (int t = 0; t < 64; ++t) sum += pv[t];
        uint8_t* atom = prow + (c >> 6) * (P_BYTES / 2);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint4 w;
          uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __half2 hv = __floats2half2_rn(pv[8 * ch + 2 * e], pv[8 * ch + 2 * e + 1]);
            pw[e] = *reinterpret_cast<uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(atom + ((ch ^ sw) << 4)) = w;
        }
      }
      l += sum;
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // epilogue: O / l after the last P.V
    if (ok && !__all_sync(0xffffffffu, mbar_wait(o_full, (nblk - 1) & 1, abort_flag))) ok = false;
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
          uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = c + 2 * e;
            const float a0 = __uint_as_float(k0 < 32 ? o0[k0] : o1[k0 - 32]);
            const float a1 = __uint_as_float(k0 + 1 < 32 ? o0[k0 + 1] : o1[k0 + 1 - 32]);
            __half2 hv = __floats2half2_rn(a0 * inv, a1 * inv);
            pw[e] = *reinterpret_cast<uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(o + c) = w;
        }
      }
    }
  }
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

cudaError_t launch_attention_tc(TcGemmCache* cache, const void* qk, const void* vt, Clips clips, void* o,
                                int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s) {
  if ((d_head != 48 && d_head != 64) || rows_pad % 8) return cudaErrorInvalidValue;
  CUtensorMap mQK, mVT;
  cudaError_t e = map2d(&mQK, qk, 64, (uint64_t)2 * n_heads * rows_pad, 64, BQ);
  if (e == cudaSuccess) e = map2d(&mVT, vt, rows_pad, (uint64_t)n_heads * 64, 64, 64);
  if (e != cudaSuccess) return e;
  AttnArgs a;
  a.clips = clips;
  a.n_heads = n_heads;
  a.d_head = d_head;
  a.rows_pad = rows_pad;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d_head);
  a.out = reinterpret_cast<__half*>(o);
  a.status = cache->status;
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((t_max + BQ - 1) / BQ, n_heads, clips.B);
  return launch_pdl(attn_tc_kernel, grid, 192, SMEM_BYTES, s, mQK, mVT, a);
}

}  // namespace gam
