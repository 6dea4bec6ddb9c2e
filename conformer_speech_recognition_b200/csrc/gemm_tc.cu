// Tensor-core GEMM for sm_100a: C = A . B^T with fused epilogues.
//
// A [M, K] fp16 (row stride lda; a strided view for the subsampling convs),
// B [N, K] fp16 weight (PyTorch Linear layout), fp32 accumulation in TMEM.
//
// Persistent, warp-specialised CTA of 320 threads, one CTA per SM:
//   warp 0      one thread issues TMA loads of 128x64 A and BNx64 B tiles
//               (128-byte swizzle) into a STAGES-deep shared-memory ring;
//   warp 1      allocates 2*BN TMEM columns (two accumulators) and one thread
//               issues tcgen05.mma (M=128, N=BN, K=16) per 16-wide K slice,
//               committing stage releases and accumulator-ready barriers;
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4) .. +31 = its 32 output rows, and one half of
//               the tile's columns, so two warps share each sub-partition and
//               hide each other's latency), bias + activation / scatter and
//               global stores, or for the residual update x += alpha (acc + b)
//               a 32 x 32 staging tile per warp that a TMA reduction adds into
//               x at the L2; then hand the accumulator back so the next tile's
//               MMAs overlap this epilogue.
// Tiles are visited n-fastest so the CTAs in flight share each A row block
// through L2 and the weight (a few MB) stays L2-resident.
// Every mbarrier wait is bounded (tc_common.cuh); a wait that gives up raises
// a CTA abort flag, the other roles stop at their next wait, in-flight copies
// and MMAs are drained with bounded waits, TMEM is freed, and a device status
// word is set for the host.
#include <cudaTypedefs.h>

#include <climits>
#include <cstdlib>
#include <cstring>

#include "gemm_tc.cuh"
#include "tc_common.cuh"

namespace gam {
namespace {

using namespace tc;

constexpr int BM = 128, BK = 64;
constexpr int A_TILE = BM * BK * 2;  // 16 KB

struct TcArgs {
  int M, N, K;
  int m_blocks, n_blocks, tiles;
  int n_split;  // output columns >= n_split read A from the second map
  int conv_c;   // 0: plain A [M, K]; else A row r = input rows 2r .. 2r+taps-1 of C = conv_c channels
  int epi;
  EpiParams ep;
  const __half* scale_t;  // INT8 weights: fp16 scales transposed to [K/64][N]
  int* status;
  uint64_t wait_ns;       // limit of every bounded wait
  int debug_skip;         // test hook: k-block counter value whose loads are not issued (-1: none)
};

// Residual epilogue: per epilogue warp two 32 x 32 fp32 staging tiles (4 KB each,
// 128-byte swizzle), used in turn, that TMA reductions add into x: a warp fills
// one while the reduction of the other is still reading it.
constexpr int kEpiWarps = 8;
constexpr int kStageTile = 32 * 32 * 4;
// Quantised-weight kernels keep one tile per warp: their shared memory goes to the
// pipeline, which their converter warps need more.
template <bool QB>
__host__ __device__ constexpr int stage_bufs() { return QB ? 1 : 2; }
template <int EPI, bool QB = false>
__host__ __device__ constexpr int epi_smem() {
  return EPI == EPI_RESID ? kEpiWarps * stage_bufs<QB>() * kStageTile : 0;
}
// Bias of the tile's columns, one 128-float copy per epilogue warp, loaded one
// tile ahead so the epilogue never waits on it.  Used by the fp16-weight kernels
// (the INT8 mainloop is bound by its converters), and by the residual epilogue
// only where it costs no pipeline stage.
constexpr int kBiasStage = 128 * 4;
constexpr int kBiasSmem = kEpiWarps * kBiasStage;
__host__ __device__ constexpr int min8(int n) { return n < 8 ? n : 8; }
// Shared memory for the operand ring: 227 KB less the epilogue staging and
// 1.25 KB of alignment slack and barriers; at most 8 stages.
template <int EPI, bool QB = false>
__host__ __device__ constexpr int ring_budget() { return 227 * 1024 - 1280 - epi_smem<EPI, QB>(); }
template <int EPI, int QBITS, int STAGE>
__host__ __device__ constexpr bool staged_bias() {
  return QBITS == 0 &&
         (EPI != EPI_RESID || min8((ring_budget<EPI>() - kBiasSmem) / STAGE) == min8(ring_budget<EPI>() / STAGE));
}

// QBITS: 0 for fp16 weights, else the bits per quantised weight (8, 6 or 4).
// MT: 128-row A tiles per CTA tile (1, or 2 for quantised weights: one converted
// B stage then feeds two accumulators, which halves the dequantisation per FLOP).
template <int BN, int QBITS, int EPI, int MT = 1>
struct Cfg {
  static constexpr bool QB = QBITS != 0;
  static constexpr int RAW_ROW = BK * QBITS / 8;             // bytes of one weight row per k-block as stored
  static constexpr int A_BYTES = MT * A_TILE;                // A tiles of one stage
  static constexpr int B_TILE = BN * BK * 2;                 // fp16 B operand (128-byte swizzle)
  static constexpr int RAW_TILE = BN * RAW_ROW;              // quantised weights as loaded (unswizzled rows)
  static constexpr int TX = A_BYTES + (QB ? RAW_TILE : B_TILE);  // bytes landed by TMA per stage
  static constexpr int STAGE = A_BYTES + B_TILE + RAW_TILE;
  static constexpr bool SB = staged_bias<EPI, QBITS, STAGE>();
  static constexpr int BIAS_SMEM = SB ? kBiasSmem : 0;
  static constexpr int STAGES = min8((ring_budget<EPI, QB>() - BIAS_SMEM) / STAGE);
  // two accumulators of MT x BN columns, rounded to a power of two
  static constexpr int ACC_COLS = MT * BN;
  static constexpr int TMEM_COLS = 2 * ACC_COLS <= 128 ? 128 : 2 * ACC_COLS <= 256 ? 256 : 512;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + epi_smem<EPI, QB>() + BIAS_SMEM + 1024 + 256;
  static_assert(MT == 1 || (QB && BN == 128), "two M tiles per CTA tile: quantised weights, 128 columns");
};

// Hardware tanh (tanh.approx, one special-function op, relative error about
// 2^-11 -- the size of the fp16 rounding the results get next).
__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Logistic function sigma(v) = (1 + tanh(v / 2)) / 2 and Swish v sigma(v).
__device__ __forceinline__ float sigm(float v) { return fmaf(0.5f, tanh_fast(0.5f * v), 0.5f); }
__device__ __forceinline__ float swish_fast(float v) {
  const float h = 0.5f * v;
  return fmaf(h, tanh_fast(h), h);
}

// 32 consecutive bias values: from the warp's shared-memory copy of the tile's
// bias (SB) or from global memory through the read-only path.
template <bool SB>
__device__ __forceinline__ void load_bias32(const float* b, float (&v)[32]) {
  const float4* p = reinterpret_cast<const float4*>(b);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 t = SB ? p[j] : __ldg(p + j);
    v[4 * j] = t.x;
    v[4 * j + 1] = t.y;
    v[4 * j + 2] = t.z;
    v[4 * j + 3] = t.w;
  }
}

// 16 values as fp16 to 32 bytes at dst (32-byte aligned) with one 256-bit store:
// a full L2 sector per thread, where two 128-bit stores would each write half of one.
__device__ __forceinline__ void store_half16(__half* dst, const float* v) {
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    __half2 h = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
    w[j] = *reinterpret_cast<uint32_t*>(&h);
  }
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Epilogue of one 32-column accumulator chunk of row r (columns n .. n+31).
template <int EPI, bool SB>
__device__ __forceinline__ void epi_chunk(const TcArgs& p, int r, int n, bool valid, const uint32_t (&u)[32],
                                          const float* bias) {
  const EpiParams& ep = p.ep;
  float v[32];
  load_bias32<SB>(bias, v);
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] += __uint_as_float(u[j]);
  switch (EPI) {
    case EPI_SWISH: {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = swish_fast(v[j]);
      __half* o = reinterpret_cast<__half*>(ep.out) + (size_t)r * ep.ldo + n;
      store_half16(o, v);
      store_half16(o + 16, v + 16);
    } break;
    case EPI_CONV1: {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = valid ? fmaxf(v[j], 0.f) : 0.f;
      __half* o = reinterpret_cast<__half*>(ep.out) + (size_t)r * ep.ldo + n;
      store_half16(o, v);
      store_half16(o + 16, v + 16);
    } break;
    case EPI_CONV2: {
      float4* px = reinterpret_cast<float4*>(ep.x + (size_t)r * ep.ldo + n);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        px[j] = valid ? make_float4(fmaxf(v[4 * j], 0.f), fmaxf(v[4 * j + 1], 0.f), fmaxf(v[4 * j + 2], 0.f),
                                    fmaxf(v[4 * j + 3], 0.f))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    } break;
    case EPI_QKV: {
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int nn = n + 16 * g;
        const int which = nn / ep.d_model;
        const int rem = nn - which * ep.d_model;
        const int h = rem / ep.d_head, cc = rem - h * ep.d_head;
        if (which < 2) {
          __half* o = reinterpret_cast<__half*>(ep.qk) + (((size_t)which * ep.n_heads + h) * ep.rows_pad + r) * 64 + cc;
          store_half16(o, v + 16 * g);
        } else {
          __half* o = reinterpret_cast<__half*>(ep.vt) + ((size_t)h * 64 + cc) * ep.rows_pad + r;
#pragma unroll
          for (int j = 0; j < 16; ++j) o[(size_t)j * ep.rows_pad] = __float2half_rn(v[16 * g + j]);
        }
      }
    } break;
    case EPI_F32: {
      float* o = reinterpret_cast<float*>(ep.out) + (size_t)r * ep.ldo + n;
      const int lim = ep.n_valid - n;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < lim) o[j] = v[j];
    } break;
    default:
      break;
  }
}

// Epilogue of this warp's half of a tile for row r: columns [half BN/2, (half+1) BN/2),
// or for the paired epilogue (GLU: 128-column blocks [value 64 | gate 64])
// the (first, second) pairs of 32-column chunks number half * BN/128 .. (half+1) * BN/128 - 1.
// bt: bias of the tile's columns (bt[c] = bias[n0 + c]), in shared memory if SB.
template <int BN, int EPI, bool SB, int NBUF>
__device__ __forceinline__ void epilogue_tile(const TcArgs& p, int r, int n0, uint32_t tbase, int half,
                                              const CUtensorMap* mX, uint8_t* stage, const float* bt,
                                              uint32_t& stage_seq) {
  const int c_lo = half * (BN / 2), c_hi = (half + 1) * (BN / 2);
  const EpiParams& ep = p.ep;
  const bool in_m = r < p.M;
  bool valid = in_m;
  if (EPI == EPI_CONV1 || EPI == EPI_CONV2) {
    if (in_m) {
      constexpr int scale = EPI == EPI_CONV1 ? 2 : 1;
      const int ci = ep.clips.find(r, scale, scale == 2 ? 2 : 0);
      const int t = r - (scale * ep.clips.e(ci) + (scale == 2 ? 2 : 0));
      valid = t >= 0 && t < (EPI == EPI_CONV1 ? ep.clips.L1(ci) : ep.clips.L2(ci));
    }
  }
  if constexpr (EPI == EPI_GLU) {
    // weight rows interleaved in blocks of 64: [value 64 | gate 64] per 128 columns
#pragma unroll 1
    for (int pr = half * (BN / 128); pr < (half + 1) * (BN / 128); ++pr) {
      const int blk = (pr >> 1) * 128, hh = (pr & 1) * 32;
      {
        uint32_t a[32], g[32];
        tmem_ld32(tbase + blk + hh, a);
        tmem_ld32(tbase + blk + 64 + hh, g);
        tmem_ld_wait();
        if (!in_m) continue;
        float bv[32], bg[32], y[32];
        load_bias32<SB>(bt + blk + hh, bv);
        load_bias32<SB>(bt + blk + 64 + hh, bg);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          y[j] = (__uint_as_float(a[j]) + bv[j]) * sigm(__uint_as_float(g[j]) + bg[j]);
        __half* o = reinterpret_cast<__half*>(ep.out) + (size_t)r * ep.ldo + (n0 + blk) / 2 + hh;
        store_half16(o, y);
        store_half16(o + 16, y + 16);
      }
    }
  } else if constexpr (EPI == EPI_RESID) {
    // x += alpha (acc + bias): this warp stages its 32 rows x 32 columns and one
    // lane hands them to a TMA reduction, so the L2 does the read-modify-write
    // of x (rows past M are clipped by the tensor map)
    const int lane = threadIdx.x & 31, row0 = r - lane;
    float bcur[32];
    load_bias32<SB>(bt + c_lo, bcur);
#pragma unroll 1
    for (int c = c_lo; c < c_hi; c += 32) {
      uint32_t u[32];
      tmem_ld32(tbase + c, u);
      float bnext[32] = {};
      if (c + 32 < c_hi) load_bias32<SB>(bt + c + 32, bnext);  // next chunk's bias while this one is read
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] = ep.alpha * (__uint_as_float(u[j]) + bcur[j]);
        bcur[j] = bnext[j];
      }
      if (row0 >= p.M) continue;
      // with two tiles, this chunk's tile was last used two chunks ago: the reductions are
      // committed in order, so waiting until at most one is still reading frees it
      if (lane == 0) {
        if (NBUF == 2) bulk_wait_read1();
        else bulk_wait_read0();
      }
      __syncwarp();
      uint8_t* buf = stage + (NBUF == 2 ? (stage_seq++ & 1) * kStageTile : 0);  // alternating across tiles too
      uint8_t* row = buf + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(row + ((j ^ (lane & 7)) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_2d(mX, buf, n0 + c, row0);
        bulk_commit();
      }
    }
  } else {
#pragma unroll 1
    for (int c = c_lo; c < c_hi; c += 32) {
      uint32_t u[32];
      tmem_ld32(tbase + c, u);
      tmem_ld_wait();
      if (in_m) epi_chunk<EPI, SB>(p, r, n0 + c, valid, u, bt + c);
    }
  }
}

// Per-warp bias of the columns this warp's epilogue reads (all 128 columns of a
// 128-wide tile, else its half of the tile), held in registers one tile ahead
// (a float4 per lane) and written to the warp's shared-memory copy when the
// tile's accumulator is ready.  Without SB the epilogue reads global memory.
template <int BN, bool SB>
struct BiasPrefetch {
  static constexpr int COLS = BN == 128 ? 128 : BN / 2;
  float* smem;
  int col0, lane;
  float4 next;
  __device__ __forceinline__ BiasPrefetch(const TcArgs& p, int half, float* s, int first_tile)
      : smem(s), col0(BN == 128 ? 0 : half * (BN / 2)), lane(threadIdx.x & 31) {
    load(p, first_tile);
  }
  __device__ __forceinline__ void load(const TcArgs& p, int tile) {
    if (SB && tile < p.tiles && lane * 4 < COLS)
      next = __ldg(reinterpret_cast<const float4*>(p.ep.bias + (tile % p.n_blocks) * BN + col0) + lane);
  }
  // bias of the tile at column n0 (bt[c] = bias[n0 + c]); starts the load for the tile after
  __device__ __forceinline__ const float* tile(const TcArgs& p, int n0, int following) {
    if (!SB) return p.ep.bias + n0;
    if (lane * 4 < COLS) reinterpret_cast<float4*>(smem)[lane] = next;
    __syncwarp();
    load(p, following);
    return smem - col0;
  }
};

constexpr int kCvtWarps = 4;  // INT8 variant: warps that dequantise the weight tile
template <bool QB>
constexpr int threads_of() { return 64 + 32 * kEpiWarps + (QB ? 32 * kCvtWarps : 0); }

// 4- and 6-bit weights are stored as u = q + 8 (resp. q + 32), in 1 .. 15 (1 .. 63),
// and laid out per 16 consecutive weights v0 .. v15 of a row so that each fp16
// pair (v_2p, v_2p+1) comes out of one shift and one mask: 32-bit word w0 holds
// the low nibbles of v0 .. v7 with v_2i in nibble i and v_2i+1 in nibble 4 + i
// (i < 4), word w1 the same for v8 .. v15; 6-bit weights add word w2 with the
// top two bits of v_2p in bits 2p .. 2p+1 and of v_2p+1 in bits 16 + 2p ..
// Writing a value u < 1024 into the mantissa of 1024.0 (fp16 0x6400) gives
// exactly 1024 + u; subtracting 1024 + the offset gives q exactly, and the
// product with the group scale is rounded once to fp16, as for INT8.
__device__ __forceinline__ uint32_t scale_pair(uint32_t u2, __half2 off, __half2 s2) {
  __half2 h = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&u2), off), s2);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void dequant16_i4(uint32_t w0, uint32_t w1, __half2 s2, uint4& out0, uint4& out1) {
  const __half2 off = __floats2half2_rn(1032.f, 1032.f);
  uint32_t o[8];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    o[p] = scale_pair(((w0 >> (4 * p)) & 0x000f000fu) | 0x64006400u, off, s2);
    o[4 + p] = scale_pair(((w1 >> (4 * p)) & 0x000f000fu) | 0x64006400u, off, s2);
  }
  out0 = make_uint4(o[0], o[1], o[2], o[3]);
  out1 = make_uint4(o[4], o[5], o[6], o[7]);
}
__device__ __forceinline__ void dequant16_i6(uint32_t w0, uint32_t w1, uint32_t w2, __half2 s2, uint4& out0,
                                             uint4& out1) {
  const __half2 off = __floats2half2_rn(1056.f, 1056.f);
  uint32_t o[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const uint32_t lo = (((p < 4 ? w0 : w1) >> (4 * (p & 3))) & 0x000f000fu);
    const uint32_t hi = ((w2 >> (2 * p)) & 0x00030003u) << 4;
    o[p] = scale_pair(lo | hi | 0x64006400u, off, s2);
  }
  out0 = make_uint4(o[0], o[1], o[2], o[3]);
  out1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// INT8 -> fp16 dequantisation of one 16-byte chunk (16 weights of one row)
// into two 16-byte chunks of the swizzled fp16 operand.  An int8 x becomes
// exactly x in fp16 by writing the byte x + 128 into the low mantissa bits of
// 1024.0 (fp16 0x6400, where the spacing is exactly 1) and subtracting 1152;
// the product with the group scale is then rounded once to fp16.
__device__ __forceinline__ void dequant16(uint4 raw, __half2 s2, uint4& out0, uint4& out1) {
  const __half2 off = __floats2half2_rn(1152.f, 1152.f);
  const uint32_t w[4] = {raw.x ^ 0x80808080u, raw.y ^ 0x80808080u, raw.z ^ 0x80808080u, raw.w ^ 0x80808080u};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo = __byte_perm(w[i], 0x64646464u, 0x4140);
    uint32_t hi = __byte_perm(w[i], 0x64646464u, 0x4342);
    __half2 hl = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&lo), off), s2);
    __half2 hh = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&hi), off), s2);
    o[2 * i] = *reinterpret_cast<uint32_t*>(&hl);
    o[2 * i + 1] = *reinterpret_cast<uint32_t*>(&hh);
  }
  out0 = make_uint4(o[0], o[1], o[2], o[3]);
  out1 = make_uint4(o[4], o[5], o[6], o[7]);
}

template <int BN, int EPI, int QBITS, int MT>
__global__ void __launch_bounds__(threads_of<QBITS != 0>(), 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
               const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mX, const TcArgs p) {
  using C = Cfg<BN, QBITS, EPI, MT>;
  constexpr bool QB = C::QB;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;                        // [STAGES][MT][A_TILE]
  uint8_t* sB = base + STAGES * C::A_BYTES;
  uint8_t* sRaw = sB + STAGES * C::B_TILE;  // INT8 variant only
  uint8_t* sEpi = base + STAGES * C::STAGE;  // residual epilogue staging, kStageBufs tiles per warp
  uint8_t* sBias = sEpi + epi_smem<EPI, QB>();  // per-warp bias copies, kBiasStage each
  uint64_t* full = reinterpret_cast<uint64_t*>(sBias + C::BIAS_SMEM);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* bready = drain + 1;  // [STAGES], INT8 variant: dequantised B tile written
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bready + STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int st = 0; st < STAGES; ++st) mbar_init(&bready[st], kCvtWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mA);
    prefetch_tmap(&mA2);
    prefetch_tmap(&mB);
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int KB = p.K / BK;
  pdl_launch_dependents();
  pdl_wait();  // the previous kernel's outputs (this GEMM's operands) are complete

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
        const int nb = tile % p.n_blocks, mb = tile / p.n_blocks;
        const int m0 = mb * BM * MT, n0 = nb * BN;
        const CUtensorMap* ma = (n0 >= p.n_split) ? &mA2 : &mA;
        for (int kb = 0; kb < KB; ++kb) {
          const int s = it % STAGES;
          if (it == p.debug_skip) {  // test hook: this stage never fills, its consumer's wait runs out
            ++it;
            continue;
          }
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          // A coordinates: plain GEMM, or tap t / channel c0 of the strided conv view,
          // read from the [pairs of input rows, 2C] map: row 2r + t = pair r + t/2, half t%2
          int ax = kb * BK, ay = m0;
          if (p.conv_c) {
            const int t = (kb * BK) / p.conv_c, c0 = kb * BK - t * p.conv_c;
            ax = (t & 1) * p.conv_c + c0;
            ay = m0 + (t >> 1);
          }
          mbar_arrive_expect_tx(&full[s], C::TX);
#pragma unroll
          for (int i = 0; i < MT; ++i) tma_load_2d(sA + s * C::A_BYTES + i * A_TILE, ma, &full[s], ax, ay + i * BM);
          if (QB) tma_load_2d(sRaw + s * C::RAW_TILE, &mB, &full[s], kb * C::RAW_ROW, n0);
          else tma_load_2d(sB + s * C::B_TILE, &mB, &full[s], kb * BK, n0);
          ++it;
        }
      }
      // every issued copy has landed before the CTA can exit (bounded)
      const int first = it > STAGES ? it - STAGES : 0;
      for (int j = first; j < it; ++j) mbar_settle(&full[j % STAGES], (j / STAGES) & 1, abort_flag, p.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN);
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * C::ACC_COLS);
        for (int kb = 0; kb < KB; ++kb) {
          const int s = it % STAGES;
          if (!mbar_wait(QB ? &bready[s] : &full[s], (it / STAGES) & 1, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = sdesc_k_sw128(smem_u32(sB + s * C::B_TILE));
#pragma unroll
          for (int i = 0; i < MT; ++i) {  // M tile i into accumulator columns [i BN, (i + 1) BN)
            const uint64_t da = sdesc_k_sw128(smem_u32(sA + s * C::A_BYTES + i * A_TILE));
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16(d + (uint32_t)(i * BN), da + 2 * k, db + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          ++it;
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      // drain: all MMAs issued by this thread complete before TMEM is freed (bounded)
      umma_commit(drain);
      mbar_settle(drain, 0, abort_flag, p.wait_ns);
    }
  } else if (QB && warp >= 2 + kEpiWarps) {
    // converter warps: quantised tile (BN rows x RAW_ROW bytes) -> fp16 swizzled operand
    // (BN rows x 128 B); each thread converts 16 weights of a row per pass
    const int t = threadIdx.x - 32 * (2 + kEpiWarps);  // 0 .. 127
    const int ch = t & 3;                              // 16-weight chunk of the row's 64
    // A thread converts rows pass * 32 + t / 4 of every tile, so the group scales of
    // its rows for the next k-block are loaded into registers one k-block ahead,
    // off the conversion's critical path.
    constexpr int NP = BN / 32;
    __half scur[NP], snext[NP];
    auto load_scales = [&](int tile, int kb, __half (&dst)[NP]) {
      if (tile >= p.tiles) return;
      const __half* sc = p.scale_t + (size_t)kb * p.N + (tile % p.n_blocks) * BN + (t >> 2);
#pragma unroll
      for (int pass = 0; pass < NP; ++pass) dst[pass] = __ldg(sc + pass * 32);
    };
    load_scales(blockIdx.x, 0, scur);
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        const int s = it % STAGES;
        if (kb + 1 < KB) load_scales(tile, kb + 1, snext);
        else load_scales(tile + gridDim.x, 0, snext);
        if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint8_t* raw = sRaw + s * C::RAW_TILE;
        uint8_t* dst = sB + s * C::B_TILE;
#pragma unroll
        for (int pass = 0; pass < NP; ++pass) {
          const int row = pass * 32 + (t >> 2);
          const uint8_t* src = raw + row * C::RAW_ROW + ch * (C::RAW_ROW / 4);
          const __half sv = scur[pass];
          uint4 o0, o1;
          if constexpr (QBITS == 8) {
            dequant16(*reinterpret_cast<const uint4*>(src), __half2(sv, sv), o0, o1);
          } else if constexpr (QBITS == 6) {
            const uint32_t* w = reinterpret_cast<const uint32_t*>(src);
            dequant16_i6(w[0], w[1], w[2], __half2(sv, sv), o0, o1);
          } else {
            const uint2 w = *reinterpret_cast<const uint2*>(src);
            dequant16_i4(w.x, w.y, __half2(sv, sv), o0, o1);
          }
          uint8_t* drow = dst + (row >> 3) * 1024 + (row & 7) * 128;
          *reinterpret_cast<uint4*>(drow + (((2 * ch) ^ (row & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(drow + (((2 * ch + 1) ^ (row & 7)) << 4)) = o1;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bready[s]);
#pragma unroll
        for (int pass = 0; pass < NP; ++pass) scur[pass] = snext[pass];
        ++it;
      }
    }
  } else {
    const int q = warp & 3;                       // TMEM lane quarter of this warp
    // MT 1: which half of the tile's columns; MT 2: which M tile (all its columns)
    const int half = (warp - 2) / 4;
    constexpr bool SB = C::SB;
    BiasPrefetch<BN, SB> bias(p, half, reinterpret_cast<float*>(sBias + (warp - 2) * kBiasStage), blockIdx.x);
    uint32_t stage_seq = 0;
    int local = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait(&tfull[acc], use & 1, abort_flag, p.wait_ns)) break;
      tc_fence_after();
      const int nb = tile % p.n_blocks, mb = tile / p.n_blocks;
      constexpr int NBUF = stage_bufs<QB>();
      uint8_t* stage = sEpi + (warp - 2) * NBUF * kStageTile;
      if constexpr (MT == 1) {
        const int r = mb * BM + q * 32 + lane;
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
        const float* bt = bias.tile(p, nb * BN, tile + gridDim.x);
        epilogue_tile<BN, EPI, SB, NBUF>(p, r, nb * BN, tbase, half, &mX, stage, bt, stage_seq);
      } else {
        const int r = mb * BM * MT + half * BM + q * 32 + lane;
        const uint32_t tbase =
            tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_COLS) + (uint32_t)(half * BN);
        const float* bt = bias.tile(p, nb * BN, tile + gridDim.x);
        epilogue_tile<BN, EPI, SB, NBUF>(p, r, nb * BN, tbase, 0, &mX, stage, bt, stage_seq);
        epilogue_tile<BN, EPI, SB, NBUF>(p, r, nb * BN, tbase, 1, &mX, stage, bt, stage_seq);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if (EPI == EPI_RESID && lane == 0) bulk_wait0();  // reductions complete before the CTA exits
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// 2-SM variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256 split as 128 rows per CTA, B split as 128
// rows per CTA).  Each CTA loads only its own 128 A rows and half of B per
// k-block (32 KB instead of 48 KB per 128x256 of output), which is what lets
// the mainloop run faster than L2 can feed the 1-SM tiles.  Both CTAs issue
// their TMA loads with completion on the leader CTA's full barrier (the
// leader expects the bytes of both); the leader alone issues the MMAs and
// commits with a two-CTA multicast to the stage / accumulator barriers of
// both CTAs; each CTA's epilogue reads its own TMEM rows and releases the
// accumulator on the leader's barrier.  No TMA load uses multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_cta(const void* p, uint32_t cta) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(cta));
  return out;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t mbar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0), "r"(0), "r"(0), "r"(0),
      "r"(0));
}
// Arrive once on the barrier at this offset in both CTAs of the pair when the MMAs complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// TN output columns per pair tile (128, 192 or 256): each CTA holds TN/2 rows of
// B per stage; two accumulators of TN columns in TMEM.
template <int TN, int EPI>
struct PairCfg {
  static constexpr int BH = TN / 2;                      // B rows per CTA
  static constexpr int B_TILE = BH * BK * 2;
  static constexpr int STAGE = A_TILE + B_TILE;
  static constexpr bool SB = staged_bias<EPI, 0, STAGE>();
  static constexpr int BIAS_SMEM = SB ? kBiasSmem : 0;
  static constexpr int STAGES = min8((ring_budget<EPI>() - BIAS_SMEM) / STAGE);
  static constexpr int TMEM_COLS = TN == 128 ? 256 : 512;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + epi_smem<EPI>() + BIAS_SMEM + 1024 + 256;
};

template <int TN, int EPI>
__global__ void __launch_bounds__(threads_of<false>(), 1)
gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
                    const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mX, const TcArgs p) {
  using C = PairCfg<TN, EPI>;
  constexpr int BN = TN, STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * A_TILE;
  uint8_t* sEpi = base + STAGES * C::STAGE;  // residual epilogue staging, kStageBufs tiles per warp
  uint8_t* sBias = sEpi + epi_smem<EPI>();    // per-warp bias copies, kBiasStage each
  uint64_t* full = reinterpret_cast<uint64_t*>(sBias + C::BIAS_SMEM);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mA);
    prefetch_tmap(&mA2);
    prefetch_tmap(&mB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive / TMA completion
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int KB = p.K / BK;
  pdl_launch_dependents();
  pdl_wait();  // the previous kernel's outputs (this GEMM's operands) are complete

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < p.tiles && ok; tile += npairs) {
        const int nb = tile % p.n_blocks, mb = tile / p.n_blocks;
        const int m0 = mb * 256 + (int)rank * 128, n0 = nb * BN;
        const CUtensorMap* ma = (n0 >= p.n_split) ? &mA2 : &mA;
        for (int kb = 0; kb < KB; ++kb) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          int ax = kb * BK, ay = m0;
          if (p.conv_c) {
            const int t = (kb * BK) / p.conv_c, c0 = kb * BK - t * p.conv_c;
            ax = (t & 1) * p.conv_c + c0;
            ay = m0 + (t >> 1);
          }
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE);
          const uint32_t fb = map_to_cta(&full[s], 0);
          tma_load_2d_pair(sA + s * A_TILE, ma, fb, ax, ay);
          tma_load_2d_pair(sB + s * C::B_TILE, &mB, fb, kb * BK, n0 + (int)rank * C::BH);
          ++it;
        }
      }
      // the leader's full barriers count both CTAs' bytes: every issued copy of
      // the pair has landed before either CTA passes the final cluster barrier
      if (leader) {
        const int first = it > STAGES ? it - STAGES : 0;
        for (int j = first; j < it; ++j) mbar_settle(&full[j % STAGES], (j / STAGES) & 1, abort_flag, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(256, BN);
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = pair; tile < p.tiles && ok; tile += npairs, ++local) {
        const int acc = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = sdesc_k_sw128(smem_u32(sA + s * A_TILE));
          const uint64_t db = sdesc_k_sw128(smem_u32(sB + s * C::B_TILE));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_f16_pair(d, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair(&empty[s]);
          ++it;
        }
        if (ok) umma_commit_pair(&tfull[acc]);
      }
      umma_commit_pair_local(drain);
      mbar_settle(drain, 0, abort_flag, p.wait_ns);
    }
  } else {
    const int q = warp & 3, half = (warp - 2) / 4;
    constexpr bool SB = C::SB;
    BiasPrefetch<BN, SB> bias(p, half, reinterpret_cast<float*>(sBias + (warp - 2) * kBiasStage), pair);
    uint32_t stage_seq = 0;
    int local = 0;
    for (int tile = pair; tile < p.tiles; tile += npairs, ++local) {
      const int acc = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait(&tfull[acc], use & 1, abort_flag, p.wait_ns)) break;
      tc_fence_after();
      const int nb = tile % p.n_blocks, mb = tile / p.n_blocks;
      const int r = mb * 256 + (int)rank * 128 + q * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const float* bt = bias.tile(p, nb * BN, tile + npairs);
      epilogue_tile<BN, EPI, SB, 2>(p, r, nb * BN, tbase, half, &mX, sEpi + (warp - 2) * 2 * kStageTile, bt,
                                    stage_seq);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_cta(&tempty[acc], 0));
    }
    if (EPI == EPI_RESID && lane == 0) bulk_wait0();  // reductions complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs (reading both CTAs' shared memory) and remote arrives are done
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, 1);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
}

// ---------------------------------------------------------------------------
// Split-K for GEMMs with few tiles (batch-1 sizes, at most 256 rows): a cluster
// of KS CTAs (2 .. 4) computes one 128 x BN tile, CTA r over the k-blocks
// [r KB/KS, (r+1) KB/KS), so KS times as many SMs stream the weights.  The
// CTAs other than the leader (rank 0) push their fp32 partial accumulators into
// the leader's shared memory (st.shared::cluster) and arrive on its barrier; the
// leader adds them to its own accumulator in rank order -- a fixed summation
// order, so the result does not depend on timing -- and runs the usual epilogue.
// One tile per cluster; no second kernel.
// ---------------------------------------------------------------------------
constexpr int kMaxSplit = 4;

template <int BN, int EPI>
struct SplitCfg {
  static constexpr int B_TILE = BN * BK * 2;
  static constexpr int STAGE = A_TILE + B_TILE;
  static constexpr int SLOT = BM * BN * 4;                 // one partial accumulator, fp32 [BM][BN]
  static constexpr int NSLOT = BN == 64 ? kMaxSplit - 1 : 1;  // KS <= 4 at 64 columns, <= 2 at 128
  static constexpr int EPI_SMEM = EPI == EPI_RESID ? kEpiWarps * kStageTile : 0;  // one staging tile per warp
  static constexpr int STAGES = min8((227 * 1024 - 1280 - EPI_SMEM - NSLOT * SLOT) / STAGE);
  static constexpr int TMEM_COLS = BN == 64 ? 64 : 128;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + (size_t)NSLOT * SLOT + EPI_SMEM + 1024 + 256;
};

__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void acc_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

template <int BN, int EPI>
__global__ void __launch_bounds__(threads_of<false>(), 1)
gemm_tc_splitk_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
                      const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mX, const TcArgs p) {
  using C = SplitCfg<BN, EPI>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * A_TILE;
  float* slots = reinterpret_cast<float*>(base + STAGES * C::STAGE);  // [NSLOT][BM][BN], filled by ranks 1..KS-1
  uint8_t* sEpi = reinterpret_cast<uint8_t*>(slots) + C::NSLOT * C::SLOT;
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::EPI_SMEM);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* parts = tfull + 1;  // leader: every partial has arrived
  uint64_t* drain = parts + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ks = (int)cluster_size(), rank = (int)cluster_rank();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(parts, (ks - 1) * kEpiWarps > 0 ? (ks - 1) * kEpiWarps : 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mA);
    prefetch_tmap(&mA2);
    prefetch_tmap(&mB);
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the leader's barriers are initialised before any remote arrive
  const uint32_t tmem = *tslot;
  pdl_launch_dependents();
  pdl_wait();

  const int tile = blockIdx.x / ks;
  const int nb = tile % p.n_blocks, mb = tile / p.n_blocks;
  const int m0 = mb * BM, n0 = nb * BN;
  const int KB = p.K / BK, kb0 = rank * KB / ks, kb1 = (rank + 1) * KB / ks;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* ma = (n0 >= p.n_split) ? &mA2 : &mA;
      int it = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, p.wait_ns)) break;
        mbar_arrive_expect_tx(&full[s], A_TILE + C::B_TILE);
        tma_load_2d(sA + s * A_TILE, ma, &full[s], kb * BK, m0);
        tma_load_2d(sB + s * C::B_TILE, &mB, &full[s], kb * BK, n0);
      }
      const int first = it > STAGES ? it - STAGES : 0;
      for (int j = first; j < it; ++j) mbar_settle(&full[j % STAGES], (j / STAGES) & 1, abort_flag, p.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN);
      bool ok = true;
      int it = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&full[s], (it / STAGES) & 1, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = sdesc_k_sw128(smem_u32(sA + s * A_TILE));
        const uint64_t db = sdesc_k_sw128(smem_u32(sB + s * C::B_TILE));
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) umma_f16(tmem, da + 2 * k, db + 2 * k, idesc, (it | k) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(tfull);
      umma_commit(drain);
      mbar_settle(drain, 0, abort_flag, p.wait_ns);
    }
  } else {
    const int q = warp & 3, half = (warp - 2) / 4;
    const int row = q * 32 + lane, r = m0 + row;
    const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
    const int c_lo = half * (BN / 2), c_hi = c_lo + BN / 2;
    bool ok = __all_sync(0xffffffffu, mbar_wait(tfull, 0, abort_flag, p.wait_ns));
    tc_fence_after();
    if (rank != 0) {
      // push this CTA's partial accumulator into slot rank - 1 of the leader
      if (ok) {
        float* slot = slots + (size_t)(rank - 1) * BM * BN + (size_t)row * BN;
        for (int c = c_lo; c < c_hi; c += 32) {
          uint32_t u[32];
          tmem_ld32(tbase + c, u);
          tmem_ld_wait();
          const uint32_t dst = map_to_cta(slot + c, 0);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_cluster_v4(dst + 16 * j, make_float4(__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                                                    __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3])));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_cta(parts, 0));  // release: the stores above come first
    } else {
      if (ks > 1 && ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(parts, 0, abort_flag, p.wait_ns));
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
      }
      // own accumulator + partials of ranks 1 .. KS-1, in that order, back into TMEM
      if (ok) {
        if (ks > 1) {
          for (int c = c_lo; c < c_hi; c += 32) {
            uint32_t u[32];
            tmem_ld32(tbase + c, u);
            tmem_ld_wait();
            for (int sidx = 0; sidx < ks - 1; ++sidx) {
              const float4* src = reinterpret_cast<const float4*>(slots + (size_t)sidx * BM * BN + (size_t)row * BN + c);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float4 v = src[j];
                u[4 * j] = __float_as_uint(__uint_as_float(u[4 * j]) + v.x);
                u[4 * j + 1] = __float_as_uint(__uint_as_float(u[4 * j + 1]) + v.y);
                u[4 * j + 2] = __float_as_uint(__uint_as_float(u[4 * j + 2]) + v.z);
                u[4 * j + 3] = __float_as_uint(__uint_as_float(u[4 * j + 3]) + v.w);
              }
            }
            acc_st32(tbase + c, u);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }
      }
      // every epilogue warp's sums are in TMEM before any epilogue reads them (the GLU
      // epilogue of one column half reads the other half's gate columns); reached by
      // all 8 epilogue warps of the leader whatever `ok` is
      tc_fence_before();
      asm volatile("bar.sync 1, %0;" ::"r"(32 * kEpiWarps) : "memory");
      tc_fence_after();
      if (ok) {
        uint32_t stage_seq = 0;
        epilogue_tile<BN, EPI, false, 1>(p, r, n0, tbase, half, &mX, sEpi + (warp - 2) * kStageTile, p.ep.bias + n0,
                                         stage_seq);
      }
      if (EPI == EPI_RESID && lane == 0) bulk_wait0();  // reductions complete before the CTA exits
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t get_encoder() {
  if (g_encode) return cudaSuccess;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return e;
  if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// 2D fp16 tensor map: `outer` rows of `inner` elements, rows `stride_bytes`
// apart, box box_inner x box_outer, 128-byte swizzle, zero fill out of bounds.
cudaError_t make_map_f16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t stride_bytes,
                         uint32_t box_inner, uint32_t box_outer) {
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (stride_bytes & 15)) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2D fp32 tensor map with 128-byte swizzle (box_inner * 4 must be 128), used for
// the residual reductions; out-of-bounds elements are neither read nor written.
cudaError_t make_map_f32(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t stride_bytes,
                         uint32_t box_inner, uint32_t box_outer) {
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (stride_bytes & 15)) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2D INT8 tensor map, no swizzle (64-byte rows of the raw weight tile).
cudaError_t make_map_i8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                        uint32_t box_outer) {
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (inner & 15)) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BN, int EPI, int QBITS, int MT = 1>
cudaError_t launch_epi(TcGemmCache* cache, const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB,
                       const CUtensorMap& mX, const TcArgs& args, cudaStream_t s) {
  using C = Cfg<BN, QBITS, EPI, MT>;
  constexpr bool QB = C::QB;
  auto kern = gemm_tc_kernel<BN, EPI, QBITS, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = args.tiles < cache->sm_count ? args.tiles : cache->sm_count;
  return launch_pdl(kern, grid, threads_of<QB>(), C::SMEM, s, mA, mA2, mB, mX, args);
}

template <int TN, int EPI>
cudaError_t launch_pair_epi(TcGemmCache* cache, const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB,
                            const CUtensorMap& mX, const TcArgs& args, cudaStream_t s) {
  using C = PairCfg<TN, EPI>;
  auto kern = gemm_tc_pair_kernel<TN, EPI>;
  static int max_clusters = 0;  // co-resident clusters of two (per process; one device model)
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(threads_of<false>());
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!max_clusters) {
    cfg.gridDim = dim3(2 * (cache->sm_count / 2));
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_clusters = n;
  }
  const int pairs = args.tiles < max_clusters ? args.tiles : max_clusters;
  cfg.gridDim = dim3(2 * pairs);
  cfg.stream = s;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kern, mA, mA2, mB, mX, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int TN>
cudaError_t launch_pair(TcGemmCache* cache, const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB,
                        const CUtensorMap& mX, const TcArgs& args, cudaStream_t s) {
  switch (args.epi) {
    case EPI_SWISH: return launch_pair_epi<TN, EPI_SWISH>(cache, mA, mA2, mB, mX, args, s);
    case EPI_GLU: return launch_pair_epi<TN, EPI_GLU>(cache, mA, mA2, mB, mX, args, s);
    case EPI_RESID: return launch_pair_epi<TN, EPI_RESID>(cache, mA, mA2, mB, mX, args, s);
    case EPI_QKV: return launch_pair_epi<TN, EPI_QKV>(cache, mA, mA2, mB, mX, args, s);
    case EPI_CONV1: return launch_pair_epi<TN, EPI_CONV1>(cache, mA, mA2, mB, mX, args, s);
    case EPI_CONV2: return launch_pair_epi<TN, EPI_CONV2>(cache, mA, mA2, mB, mX, args, s);
    case EPI_F32: return launch_pair_epi<TN, EPI_F32>(cache, mA, mA2, mB, mX, args, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN, int QBITS, int MT = 1>
cudaError_t launch_bn(TcGemmCache* cache, const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB,
                      const CUtensorMap& mX, const TcArgs& args, cudaStream_t s) {
  switch (args.epi) {
    case EPI_SWISH: return launch_epi<BN, EPI_SWISH, QBITS, MT>(cache, mA, mA2, mB, mX, args, s);
    case EPI_GLU: return launch_epi<BN, EPI_GLU, QBITS, MT>(cache, mA, mA2, mB, mX, args, s);
    case EPI_RESID: return launch_epi<BN, EPI_RESID, QBITS, MT>(cache, mA, mA2, mB, mX, args, s);
    case EPI_QKV: return launch_epi<BN, EPI_QKV, QBITS, MT>(cache, mA, mA2, mB, mX, args, s);
    case EPI_F32: return launch_epi<BN, EPI_F32, QBITS, MT>(cache, mA, mA2, mB, mX, args, s);
    case EPI_CONV1:
      if constexpr (QBITS == 0) return launch_epi<BN, EPI_CONV1, 0>(cache, mA, mA2, mB, mX, args, s);
      return cudaErrorInvalidValue;  // the subsampling convs keep fp16 weights
    case EPI_CONV2:
      if constexpr (QBITS == 0) return launch_epi<BN, EPI_CONV2, 0>(cache, mA, mA2, mB, mX, args, s);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <int QBITS>
cudaError_t launch_width(int BN, int mt, TcGemmCache* cache, const CUtensorMap& mA, const CUtensorMap& mA2,
                         const CUtensorMap& mB, const CUtensorMap& mX, const TcArgs& args, cudaStream_t s) {
  if (BN == 64) {  // narrow tiles: fp16 weights and few rows only
    if constexpr (QBITS == 0) return launch_bn<64, 0>(cache, mA, mA2, mB, mX, args, s);
    return cudaErrorInvalidValue;
  }
  if (mt == 2) {  // two M tiles per converted B stage: quantised weights, 128 columns
    if constexpr (QBITS != 0) {
      if (BN == 128) return launch_bn<128, QBITS, 2>(cache, mA, mA2, mB, mX, args, s);
    }
    return cudaErrorInvalidValue;
  }
  if (BN == 256) return launch_bn<256, QBITS>(cache, mA, mA2, mB, mX, args, s);
  if (BN == 192) return launch_bn<192, QBITS>(cache, mA, mA2, mB, mX, args, s);
  return launch_bn<128, QBITS>(cache, mA, mA2, mB, mX, args, s);
}

template <int BN, int EPI>
cudaError_t launch_split_epi(const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB,
                             const CUtensorMap& mX, const TcArgs& args, int ks, cudaStream_t s) {
  using C = SplitCfg<BN, EPI>;
  auto kern = gemm_tc_splitk_kernel<BN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(args.tiles * ks);
  cfg.blockDim = dim3(threads_of<false>());
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kern, mA, mA2, mB, mX, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_split(int BN, const CUtensorMap& mA, const CUtensorMap& mA2, const CUtensorMap& mB,
                         const CUtensorMap& mX, const TcArgs& args, int ks, cudaStream_t s) {
  if (BN == 128) {
    if (args.epi == EPI_GLU) return launch_split_epi<128, EPI_GLU>(mA, mA2, mB, mX, args, ks, s);
    return cudaErrorInvalidValue;
  }
  switch (args.epi) {
    case EPI_SWISH: return launch_split_epi<64, EPI_SWISH>(mA, mA2, mB, mX, args, ks, s);
    case EPI_RESID: return launch_split_epi<64, EPI_RESID>(mA, mA2, mB, mX, args, ks, s);
    case EPI_QKV: return launch_split_epi<64, EPI_QKV>(mA, mA2, mB, mX, args, ks, s);
    case EPI_F32: return launch_split_epi<64, EPI_F32>(mA, mA2, mB, mX, args, ks, s);
    default: return cudaErrorInvalidValue;
  }
}

// Split count for a GEMM of few rows: the largest KS in 2 .. 4 (2 for the GLU's
// 128-column tiles) that divides the k-blocks and leaves each CTA at least two
// of them (forced), or -- chosen by the library -- at least eight, with tiles x KS
// within the SMs.  Measured at batch 1 (d768): the cluster's fixed cost (launch,
// partial-sum exchange) pays off only for deep K (FFN down, K = 3072: 0.73 ->
// 0.67 ms per step); at K = 768 a split made FFN up, QKV and the output
// projection slower.  0 when none applies.
int split_count(const TcGemmCache* cache, int M, int N, int K, int bn, bool forced) {
  const int tiles = ((M + BM - 1) / BM) * (N / bn);
  const int KB = K / BK;
  for (int c = bn == 64 ? kMaxSplit : 2; c >= 2; --c)
    if (KB % c == 0 && (forced ? KB / c >= 2 : (KB / c >= 8 && tiles * c <= cache->sm_count))) return c;
  return 0;
}

}  // namespace

bool tc_supported(int a_dtype, int b_dtype, int N, int K, int epi) {
  return a_dtype == 1 && b_dtype >= 1 && b_dtype <= 4 && N % 256 == 0 && K % 64 == 0 && K >= 64 &&
         (epi == EPI_SWISH || epi == EPI_GLU || epi == EPI_RESID || epi == EPI_QKV || epi == EPI_CONV1 ||
          epi == EPI_CONV2 || epi == EPI_F32);
}

cudaError_t tc_init(TcGemmCache* cache, int device) {
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&cache->sm_count, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return e;
  // GAM_GEMM_TILES=single|pair|auto (default auto): tile-shape policy of the fp16 GEMMs
  if (const char* v = std::getenv("GAM_GEMM_TILES")) {
    if (!std::strcmp(v, "single")) cache->pair_mode = 0;
    else if (!std::strcmp(v, "pair")) cache->pair_mode = 2;
    else cache->pair_mode = 1;
  }
  // GAM_SPLITK=0: no split-K for GEMMs of few rows
  if (const char* v = std::getenv("GAM_SPLITK")) cache->splitk = std::strcmp(v, "0") != 0;
  // GAM_QB_TILES=m1|m2 (default m2): M tiles per CTA tile of the quantised-weight GEMMs
  if (const char* v = std::getenv("GAM_QB_TILES")) cache->qb_mt = std::strcmp(v, "m1") ? 2 : 1;
  e = cudaMalloc(&cache->status, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemset(cache->status, 0, sizeof(int));
}

// Relative cost per output column of a paired-CTA tile against a single-CTA
// tile of the same width: each SM of a pair loads half as much of B, which the
// mainloop turns into speed because it is bound by the L2 -> shared memory feed.
constexpr double kPairCost = 0.7;
// Weight of the round-up to whole waves: with fp16 weights a partly filled last
// wave runs faster per tile than a full one (fewer SMs share the L2 feed), so
// tiles count for 0.75 x (tiles / units) + 0.25 x ceil(tiles / units) waves.
// The INT8 mainloop is bound by its converter warps inside each SM instead, and
// its waves count whole.
constexpr double kWaveRoundUp = 0.25;

// Tile shape: over single-CTA tiles (128 rows) and paired-CTA tiles (256 rows
// on two SMs) of width 256, 192 or 128 dividing N (the GLU epilogue needs
// 128-column blocks), the one that minimises (waves of tiles over the SMs) x
// (per-SM tile cost), counting a fixed per-tile overhead of 32 columns.  The
// constants were fitted to measured times of the encoder's GEMM shapes on B200.
// variant: -1 any, 0 single-CTA only, 1 paired-CTA only; width 0: any.  With a
// second A operand from column n_split on (n_split > 0), tiles may not straddle it.
TileShape choose_tile(const TcGemmCache* cache, int M, int N, int epi, bool qb, int variant, int width,
                      int n_split) {
  TileShape best{false, 0};
  double best_cost = 1e30;
  const int sms = cache->sm_count;
  for (int pair = 0; pair < 2; ++pair) {
    if ((variant >= 0 && pair != variant) || (pair && qb)) continue;
    if (variant < 0 && ((pair && cache->pair_mode == 0) || (!pair && cache->pair_mode == 2))) continue;
    const int units = pair ? sms / 2 : sms;
    const int mt = pair ? (M + 255) / 256 : (M + BM - 1) / BM;
    for (int bn : {256, 192, 128, 64}) {
      if (N % bn || (width && bn != width) || (n_split > 0 && n_split % bn)) continue;
      // 64-column tiles spread a weight matrix over more SMs when the rows are few
      // (batch-1 latency); single-CTA, fp16 weights, at most 256 rows
      if (bn == 64 && (pair || qb || epi == EPI_GLU || M > 256)) continue;
      if (epi == EPI_GLU && bn % 128) continue;
      const int tiles = mt * (N / bn);
      const double round_up = qb ? 1.0 : kWaveRoundUp;
      const double waves = round_up * (double)((tiles + units - 1) / units) + (1.0 - round_up) * (double)tiles / units;
      const double cost = waves * (bn + 32) * (pair ? kPairCost : 1.0);
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = TileShape{pair != 0, bn};
      }
    }
  }
  // the "pair" policy falls back to single-CTA tiles where no paired tile applies
  if (!best.width && variant < 0 && cache->pair_mode == 2) return choose_tile(cache, M, N, epi, qb, 0, width, n_split);
  // Quantised weights: 256 x 128 tiles whose converted B stage feeds two 128-row
  // accumulators, unless a width other than 128 was asked for or the context
  // selected one M tile per CTA tile (GAM_QB_TILES=m1).  Their converter warps, not
  // the tensor core, bound these GEMMs, so halving the dequantisation per FLOP
  // outweighs the coarser tiles.
  if (qb && cache->qb_mt == 2 && variant <= 0 && (width == 0 || width == 128) && N % 128 == 0 &&
      (n_split <= 0 || n_split % 128 == 0))
    return TileShape{false, 128, 2};
  return best;
}

cudaError_t launch_gemm_tc(TcGemmCache* cache, const void* A, const void* A2, int n_split, int lda, WeightOp B, int M,
                           int N, int K, int epi, const EpiParams& ep, cudaStream_t s, int variant, int width) {
  if (!tc_supported(1, B.dtype, N, K, epi) || M <= 0) return cudaErrorInvalidValue;
  // fp16 outputs are written 32 bytes per thread: 32-byte aligned rows
  if ((epi == EPI_SWISH || epi == EPI_GLU || epi == EPI_CONV1) &&
      ((reinterpret_cast<uintptr_t>(ep.out) & 31) || ep.ldo % 16))
    return cudaErrorInvalidValue;
  if (epi == EPI_QKV && ((reinterpret_cast<uintptr_t>(ep.qk) & 31) || ep.d_head % 16)) return cudaErrorInvalidValue;
  const bool qb = B.dtype >= 2;  // INT8 / INT6 / INT4 g64 weights: dequantised in the mainloop
  const int qbits = B.dtype == 2 ? 8 : B.dtype == 3 ? 6 : 4;
  if (qb && !B.scale_t) return cudaErrorInvalidValue;
  // Few rows (batch-1 sizes): split K over a cluster when that multiplies the SMs
  // streaming the weights (variant 2 forces it).  fp16 weights, plain A operand.
  if (variant == 2 || (variant < 0 && width == 0 && cache->splitk && M <= 256)) {
    const int bn = epi == EPI_GLU ? 128 : 64;
    const bool fits = B.dtype == 1 && lda >= K && M <= 256 && N % bn == 0 && (!A2 || n_split % bn == 0) &&
                      (epi == EPI_SWISH || epi == EPI_GLU || epi == EPI_RESID || epi == EPI_QKV || epi == EPI_F32);
    const int ks = fits ? split_count(cache, M, N, K, bn, variant == 2) : 0;
    if (ks >= 2) {
      CUtensorMap mA, mA2, mB, mX;
      cudaError_t e = make_map_f16(&mA, A, K, M, (uint64_t)lda * 2, BK, BM);
      if (e == cudaSuccess) e = make_map_f16(&mA2, A2 ? A2 : A, K, M, (uint64_t)lda * 2, BK, BM);
      if (e == cudaSuccess) e = make_map_f16(&mB, B.w, K, N, (uint64_t)K * 2, BK, bn);
      mX = mB;
      if (e == cudaSuccess && epi == EPI_RESID) e = make_map_f32(&mX, ep.x, N, M, (uint64_t)ep.ldo * 4, 32, 32);
      if (e != cudaSuccess) return e;
      TcArgs args;
      args.M = M;
      args.N = N;
      args.K = K;
      args.m_blocks = (M + BM - 1) / BM;
      args.n_blocks = N / bn;
      args.tiles = args.m_blocks * args.n_blocks;
      args.n_split = A2 ? n_split : INT_MAX;
      args.conv_c = 0;
      args.epi = epi;
      args.ep = ep;
      args.scale_t = nullptr;
      args.status = cache->status;
      args.wait_ns = cache->debug_limit_ns ? cache->debug_limit_ns : kWaitLimitNs;
      args.debug_skip = -1;
      cache->debug_limit_ns = 0;
      cache->debug_skip = -1;
      return launch_split(bn, mA, mA2, mB, mX, args, ks, s);
    }
    if (variant == 2) return cudaErrorInvalidValue;  // forced, but no split applies
  }
  const TileShape t = choose_tile(cache, M, N, epi, qb, variant, width, A2 ? n_split : 0);
  if (!t.width) return cudaErrorInvalidValue;
  const bool pair = t.pair;
  const int BN = t.width, mt = t.mt;
  // lda < K: stride-2 convolution view (lda = 2C, K = taps * C, C % 64 == 0); the
  // buffer behind it holds (M + 2) * lda elements, mapped as M + 2 rows of 2C.
  const bool conv = lda < K;
  if (conv && ((lda & 1) || (lda / 2) % BK || K % (lda / 2))) return cudaErrorInvalidValue;
  CUtensorMap mA, mA2, mB;
  cudaError_t e = conv ? make_map_f16(&mA, A, lda, (uint64_t)M + 2, (uint64_t)lda * 2, BK, BM)
                       : make_map_f16(&mA, A, K, M, (uint64_t)lda * 2, BK, BM);
  if (e == cudaSuccess && !conv) e = make_map_f16(&mA2, A2 ? A2 : A, K, M, (uint64_t)lda * 2, BK, BM);
  if (conv) mA2 = mA;
  if (e == cudaSuccess)
    e = qb ? make_map_i8(&mB, B.w, (uint64_t)K * qbits / 8, N, BK * qbits / 8, BN)
           : make_map_f16(&mB, B.w, K, N, (uint64_t)K * 2, BK, pair ? (uint32_t)(BN / 2) : (uint32_t)BN);
  if (e != cudaSuccess) return e;
  TcArgs args;
  args.M = M;
  args.N = N;
  args.K = K;
  args.m_blocks = (pair || mt == 2) ? (M + 255) / 256 : (M + BM - 1) / BM;
  args.n_blocks = N / BN;
  args.tiles = args.m_blocks * args.n_blocks;
  args.n_split = A2 ? n_split : INT_MAX;
  args.conv_c = conv ? lda / 2 : 0;
  args.epi = epi;
  args.ep = ep;
  args.scale_t = B.scale_t;
  args.status = cache->status;
  args.wait_ns = cache->debug_limit_ns ? cache->debug_limit_ns : kWaitLimitNs;
  args.debug_skip = pair ? -1 : cache->debug_skip;
  cache->debug_limit_ns = 0;  // the hook applies to one launch
  cache->debug_skip = -1;
  // residual epilogue: fp32 map over x [M, N] (row stride ldo) for the TMA reduction
  CUtensorMap mX = mB;
  if (epi == EPI_RESID) {
    e = make_map_f32(&mX, ep.x, N, M, (uint64_t)ep.ldo * 4, 32, 32);
    if (e != cudaSuccess) return e;
  }
  if (pair) {
    if (BN == 256) return launch_pair<256>(cache, mA, mA2, mB, mX, args, s);
    if (BN == 192) return launch_pair<192>(cache, mA, mA2, mB, mX, args, s);
    return launch_pair<128>(cache, mA, mA2, mB, mX, args, s);
  }
  if (B.dtype == 2) return launch_width<8>(BN, mt, cache, mA, mA2, mB, mX, args, s);
  if (B.dtype == 3) return launch_width<6>(BN, mt, cache, mA, mA2, mB, mX, args, s);
  if (B.dtype == 4) return launch_width<4>(BN, mt, cache, mA, mA2, mB, mX, args, s);
  return launch_width<0>(BN, 1, cache, mA, mA2, mB, mX, args, s);
}

cudaError_t launch_attention(TcGemmCache* cache, const void* qk, const void* vt, Clips clips, void* o, int t_half,
                             int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s) {
  // GAM_ATTN=1 selects the earlier 128-key kernel (read at each launch)
  const char* form = std::getenv("GAM_ATTN");
  const bool first_form = form && std::strcmp(form, "1") == 0;
  if (t_half && !first_form) return launch_attention_tc2(cache, qk, vt, clips, o, rows_pad, n_heads, d_head, t_max, s);
  if (t_half) return launch_attention_tc(cache, qk, vt, clips, o, rows_pad, n_heads, d_head, t_max, s);
  return launch_attention_simt(qk, vt, clips, o, t_half, rows_pad, n_heads, d_head, t_max, s);
}

cudaError_t tc_read_status(TcGemmCache* c, int* st) {
  *st = 0;
  if (!c->status) return cudaSuccess;
  return cudaMemcpy(st, c->status, sizeof(int), cudaMemcpyDeviceToHost);
}
cudaError_t tc_reset_status(TcGemmCache* c) {
  if (!c->status) return cudaSuccess;
  return cudaMemset(c->status, 0, sizeof(int));
}
void tc_release(TcGemmCache* c) {
  if (c->status) cudaFree(c->status);
  c->status = nullptr;
}

}  // namespace gam
