// Memory-bound row kernels of the Conformer block and the CTC decoder.
//
//  * LayerNorm over d (one warp per row, float4 loads, two-pass statistics in
//    registers), in three forms: plain; fused with the rotary embedding of
//    "GigaAM on MLX: the transcripts matched, but the model was broken",
//    "Trap 2" (u = LN(x) feeds V, u_rot = u * cos + rotate_half(u) * sin per
//    head feeds Q and K; tables of base 5000 from "Trap 1"); and chained
//    (block-final LayerNorm written back to the residual stream, then the next
//    block's first LayerNorm).
//  * Depthwise conv over time with BatchNorm folded into its weights and
//    bias, then Swish (textbook Conformer convolution module), rows outside
//    the clip read as zero.
//  * Encoder output scatter to the padded [B, T', d] layout.
//  * CTC: log-softmax + first-index argmax per frame, then greedy collapse
//    (runs merged, blanks dropped) with a block-wide scan.
#include <algorithm>

#include "common.cuh"
#include "tc_common.cuh"

namespace gam {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
template <>
__device__ __forceinline__ void store4<__half>(__half* p, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ float ld1(const float* p) { return *p; }
__device__ __forceinline__ float ld1(const __half* p) { return __half2float(*p); }

// Normalise the row held in v[0..NV) (float4 chunks, chunk j at column 4(32 j + lane)),
// NV = d / 128 fixed at compile time so only the registers of one row are live.
template <int NV>
__device__ __forceinline__ void ln_row(float4 (&v)[NV], int d, float eps, const float* g, const float* b, int lane) {
  constexpr int nv = NV;
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < nv; ++j) s += v[j].x + v[j].y + v[j].z + v[j].w;
  const float mean = warp_sum(s) / d;
  float q = 0.f;
#pragma unroll
  for (int j = 0; j < nv; ++j) {
      v[j].x -= mean; v[j].y -= mean; v[j].z -= mean; v[j].w -= mean;
      q += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
    }
  const float rstd = rsqrtf(warp_sum(q) / d + eps);
#pragma unroll
  for (int j = 0; j < nv; ++j) {
      const int c = (j * 32 + lane) * 4;
      const float4 gg = *reinterpret_cast<const float4*>(g + c);
      const float4 bb = *reinterpret_cast<const float4*>(b + c);
      v[j].x = v[j].x * rstd * gg.x + bb.x;
      v[j].y = v[j].y * rstd * gg.y + bb.y;
      v[j].z = v[j].z * rstd * gg.z + bb.z;
      v[j].w = v[j].w * rstd * gg.w + bb.w;
    }
}

template <int NV>
__device__ __forceinline__ void load_row(const float* x, float4 (&v)[NV], int lane) {
#pragma unroll
  for (int j = 0; j < NV; ++j) v[j] = *reinterpret_cast<const float4*>(x + (j * 32 + lane) * 4);
}

// The LayerNorm kernels run one resident wave of CTAs (grid sized from the
// occupancy); warp w of the grid takes rows w, w + W, w + 2W, ... (W warps in
// the grid) and loads its next row while it normalises the current one, so
// each SM keeps a row per warp in flight and no second, partly filled wave
// follows the first.

// Plain LayerNorm.
template <typename T, int NV>
__global__ void __launch_bounds__(256)
ln_kernel(const float* __restrict__ x, const float* __restrict__ g, const float* __restrict__ b, float eps,
          T* __restrict__ u, int rows) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int d = NV * 128;
  const int lane = threadIdx.x & 31, nw = gridDim.x * 8;
  int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  float4 cur[NV], nxt[NV];
  if (row < rows) load_row<NV>(x + (size_t)row * d, cur, lane);
  for (; row < rows; row += nw) {
    if (row + nw < rows) load_row<NV>(x + (size_t)(row + nw) * d, nxt, lane);
    ln_row<NV>(cur, d, eps, g, b, lane);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      store4<T>(u + (size_t)row * d + (j * 32 + lane) * 4, cur[j]);
      cur[j] = nxt[j];
    }
  }
}

// Two LayerNorms in a row (a block's final norm, then the next block's first):
// x <- LN1(x) in place, u = LN2(LN1(x)).
template <typename T, int NV>
__global__ void __launch_bounds__(256)
ln_chain_kernel(float* __restrict__ x, const float* __restrict__ g1, const float* __restrict__ b1,
                const float* __restrict__ g2, const float* __restrict__ b2, float eps, T* __restrict__ u, int rows) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int d = NV * 128;
  const int lane = threadIdx.x & 31, nw = gridDim.x * 8;
  int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  float4 cur[NV], nxt[NV];
  if (row < rows) load_row<NV>(x + (size_t)row * d, cur, lane);
  for (; row < rows; row += nw) {
    if (row + nw < rows) load_row<NV>(x + (size_t)(row + nw) * d, nxt, lane);
    float* xr = x + (size_t)row * d;
    T* ur = u + (size_t)row * d;
    ln_row<NV>(cur, d, eps, g1, b1, lane);
#pragma unroll
    for (int j = 0; j < NV; ++j) *reinterpret_cast<float4*>(xr + (j * 32 + lane) * 4) = cur[j];
    ln_row<NV>(cur, d, eps, g2, b2, lane);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      store4<T>(ur + (j * 32 + lane) * 4, cur[j]);
      cur[j] = nxt[j];
    }
  }
}

// LayerNorm, then RoPE on the normalised row: u = LN(x) and, per head,
// urot = u cos(t w_i) + rotate_half(u) sin(t w_i) at the row's position t in
// its clip.  The row goes through shared memory so each lane can read the
// partner half of its columns; the cos / sin tables are [T][d_head / 2].
template <typename T, int DH, int NV>
__global__ void __launch_bounds__(256)
ln_rope_kernel(const float* __restrict__ x, const float* __restrict__ g, const float* __restrict__ b, float eps,
               const float* __restrict__ cos_tab, const float* __restrict__ sin_tab, Clips clips, T* __restrict__ u,
               T* __restrict__ urot, int rows) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int dh = DH, half = DH / 2, d = NV * 128;
  static_assert(half % 4 == 0, "a float4 of columns never straddles a half head");
  __shared__ __align__(16) float srow[8][d];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = gridDim.x * 8;
  float* sr = srow[w];
  int row = blockIdx.x * 8 + w;
  float4 cur[NV], nxt[NV];
  if (row < rows) load_row<NV>(x + (size_t)row * d, cur, lane);
  for (; row < rows; row += nw) {
    if (row + nw < rows) load_row<NV>(x + (size_t)(row + nw) * d, nxt, lane);
    ln_row<NV>(cur, d, eps, g, b, lane);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * 32 + lane) * 4;
      store4<T>(u + (size_t)row * d + c, cur[j]);
      *reinterpret_cast<float4*>(sr + c) = cur[j];
      cur[j] = nxt[j];
    }
    __syncwarp();
    const int ci = clips.find(row, 1, 0);
    int t = row - clips.e(ci);
    if (t < 0 || t >= clips.L2(ci)) t = 0;  // gap row: any finite rotation
    const float* ct = cos_tab + (size_t)t * half;
    const float* st = sin_tab + (size_t)t * half;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c0 = (j * 32 + lane) * 4;
      const int cc = c0 % dh;
      const bool first = cc < half;
      const int i = first ? cc : cc - half;
      const float4 cs = __ldg(reinterpret_cast<const float4*>(ct + i));
      const float4 sn = __ldg(reinterpret_cast<const float4*>(st + i));
      const float4 a = *reinterpret_cast<const float4*>(sr + c0);
      const float4 q = *reinterpret_cast<const float4*>(sr + (first ? c0 + half : c0 - half));
      const float sg = first ? -1.f : 1.f;  // rotate_half: [-x2, x1]
      store4<T>(urot + (size_t)row * d + c0,
                make_float4(fmaf(sg * q.x, sn.x, a.x * cs.x), fmaf(sg * q.y, sn.y, a.y * cs.y),
                            fmaf(sg * q.z, sn.z, a.z * cs.z), fmaf(sg * q.w, sn.w, a.w * cs.w)));
    }
    __syncwarp();  // the row buffer is rewritten by the next iteration
  }
}

// Swish: exact form for the fp32 build mode; in the fp16 modes one hardware
// tanh (relative error ~2^-11, the size of the fp16 rounding of the result).
template <typename T>
__device__ __forceinline__ float swish_t(float v) {
  if constexpr (sizeof(T) == 2) {
    const float h = 0.5f * v;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
  } else {
    return v / (1.f + expf(-v));
  }
}

// Depthwise conv + folded BatchNorm + Swish.  CTA = 64 rows x 128 channels,
// 256 threads: thread (channel c, row half h) produces rows 32h .. 32h+31 of
// channel c in 4 groups of 8, sliding over the staged input rows so each
// shared-memory value feeds up to 8 outputs.  Weights (tap-major [K][d], BN
// folded) live in registers.  Clip bounds are looked up once per row; groups
// whose whole window lies inside one clip take the plain path, the others
// repeat it once per clip among their rows with out-of-clip inputs zeroed.
template <typename T, int K>
__global__ void __launch_bounds__(256)
dwconv_kernel(const T* __restrict__ g, const float* __restrict__ w, const float* __restrict__ bias, Clips clips,
              T* __restrict__ out, int rows, int d) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int PAD = (K - 1) / 2, R = 64, HALO = R + 2 * PAD;
  __shared__ __align__(16) float tile[HALO][128];
  __shared__ int s_lo[R], s_hi[R];
  const int r0 = blockIdx.x * R, c0 = blockIdx.y * 128;
  // staging: one warp per row, 4 channels per lane, one 16-byte shared store each
  // (conflict-free); every load of the thread is issued before the first store
  constexpr int ITEMS = (HALO * 32 + 255) / 256;
  float4 v[ITEMS];
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = threadIdx.x + it * 256;
    const int rr = idx >> 5, c4 = (idx & 31) * 4;
    const int src = r0 - PAD + rr;
    v[it] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (idx < HALO * 32 && src >= 0 && src < rows) {
      if constexpr (sizeof(T) == 2) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(g + (size_t)src * d + c0 + c4));
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
        v[it] = make_float4(a.x, a.y, b.x, b.y);
      } else {
        v[it] = __ldg(reinterpret_cast<const float4*>(g + (size_t)src * d + c0 + c4));
      }
    }
  }
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const int idx = threadIdx.x + it * 256;
    if (idx < HALO * 32) *reinterpret_cast<float4*>(&tile[idx >> 5][(idx & 31) * 4]) = v[it];
  }
  if (threadIdx.x < R) {
    const int r = r0 + threadIdx.x;
    int lo = 0, hi = 0;
    if (r < rows) {
      const int ci = clips.find(r, 1, 0);
      lo = clips.e(ci);
      hi = lo + clips.L2(ci);
    }
    s_lo[threadIdx.x] = lo;
    s_hi[threadIdx.x] = hi;
  }
  __syncthreads();
  const int cc = threadIdx.x & 127, c = c0 + cc;
  float wk[K];
#pragma unroll
  for (int k = 0; k < K; ++k) wk[k] = __ldg(w + (size_t)k * d + c);
  const float bv = __ldg(bias + c);
  const int rbase = (threadIdx.x >> 7) * 32;
#pragma unroll 1
  for (int grp = 0; grp < 4; ++grp) {
    const int j0 = rbase + grp * 8;  // first tile row of this group
    const int lo = s_lo[j0], hi = s_hi[j0];
    const bool same = s_lo[j0 + 7] == lo;
    const int r = r0 + j0;
    float acc[8];
    if (same && r - PAD >= lo && r + 7 + PAD < hi) {
      // interior: every tap of the 8 rows is inside the clip
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = bv;
#pragma unroll
      for (int t = 0; t < K + 7; ++t) {
        const float x = tile[j0 + t][cc];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int k = t - i;
          if (k >= 0 && k < K) acc[i] = fmaf(wk[k], x, acc[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = swish_t<T>(acc[i]);
    } else {
      // near a clip edge: the group's rows fall into runs of the same clip (rows of
      // a clip are contiguous); each run takes the interior computation over the
      // window with the input rows outside its clip read as zero
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      int i0 = 0;
#pragma unroll 1
      while (i0 < 8) {
        const int li = s_lo[j0 + i0], hiI = s_hi[j0 + i0];
        int i1 = i0 + 1;
        while (i1 < 8 && s_lo[j0 + i1] == li) ++i1;
        const unsigned span = (unsigned)(hiI - li);
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = bv;
#pragma unroll
        for (int t = 0; t < K + 7; ++t) {
          const float xm = ((unsigned)(r - PAD + t - li) < span) ? tile[j0 + t][cc] : 0.f;  // input row r - PAD + t
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int k = t - i;
            if (k >= 0 && k < K) a[i] = fmaf(wk[k], xm, a[i]);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i >= i0 && i < i1 && (unsigned)(r + i - li) < span) acc[i] = swish_t<T>(a[i]);
        i0 = i1;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (r + i >= rows) break;
      if constexpr (sizeof(T) == 2) out[(size_t)(r + i) * d + c] = __float2half_rn(acc[i]);
      else out[(size_t)(r + i) * d + c] = acc[i];
    }
  }
}

// Packed fp32 (sm_100 f32x2): a 64-bit register holds the values of two adjacent
// channels, and one fma.rn.f32x2 does both channels' multiply-add.
__device__ __forceinline__ unsigned long long pk2(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 upk2(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// fp16 activations, persistent and TMA-fed.  Work items are (64 rows, 128
// channels) tiles; each CTA walks its items with a ring of kDwStages tiles in
// shared memory that one thread fills by TMA (halo rows included: a negative or
// past-the-end row coordinate reads zeros), so the load of the next tiles needs
// no registers and overlaps this tile's arithmetic, which reads the fp16 tile
// directly: each thread owns two adjacent channels and 16 rows in 2 groups of 8,
// one packed fma.rn.f32x2 per tap for both channels (one fp32 fma per channel, in
// tap order), BN folded; a group of 8 rows that meets a clip edge runs once per
// clip among its rows with the inputs outside that clip zeroed.  Waits are bounded; a wait that gives up sets `status`.
constexpr int kDwStages = 2;

template <int K>
__global__ void __launch_bounds__(256, 2)
dwconv_tma_kernel(const __grid_constant__ CUtensorMap mG, const float* __restrict__ w, const float* __restrict__ bias,
                  Clips clips, __half* __restrict__ out, int rows, int d, int n_items, int* status) {
  using namespace tc;
  constexpr int PAD = (K - 1) / 2, R = 64, HALO = R + 2 * PAD;
  constexpr uint32_t TILE_BYTES = HALO * 128 * 2;
  extern __shared__ __align__(128) uint8_t dw_smem[];
  // [kDwStages][HALO][128]; rows of 256 B keep every stage 128-byte aligned
  __half* tiles = reinterpret_cast<__half*>((reinterpret_cast<uintptr_t>(dw_smem) + 127) & ~(uintptr_t)127);
  __shared__ uint64_t full[kDwStages];
  __shared__ int s_lo[R], s_hi[R];
  __shared__ int s_abort;
  const int n_cb = d / 128;
  if (threadIdx.x == 0) {
    prefetch_tmap(&mG);
    for (int i = 0; i < kDwStages; ++i) mbar_init(&full[i], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();
  volatile int* abort_flag = &s_abort;
  auto issue = [&](int it) {  // item number it of this CTA into stage it % kDwStages
    const int item = blockIdx.x + it * gridDim.x;
    if (item >= n_items) return;
    const int st = it % kDwStages;
    mbar_arrive_expect_tx(&full[st], TILE_BYTES);
    tma_load_2d(tiles + (size_t)st * HALO * 128, &mG, &full[st], (item % n_cb) * 128, (item / n_cb) * R - PAD);
  };
  if (threadIdx.x == 0)
    for (int it = 0; it < kDwStages; ++it) issue(it);
  const int cc = 2 * (threadIdx.x & 63);
  const int rbase = (threadIdx.x >> 6) * 16;
  int cur_cb = -1;
  unsigned long long wk[K], bv = 0;
  int it = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
    const int cb = item % n_cb, r0 = (item / n_cb) * R, c = cb * 128 + cc;
    const int st = it % kDwStages;
    if (threadIdx.x < R) {
      const int r = r0 + threadIdx.x;
      int lo = 0, hi = 0;
      if (r < rows) {
        const int ci = clips.find(r, 1, 0);
        lo = clips.e(ci);
        hi = lo + clips.L2(ci);
      }
      s_lo[threadIdx.x] = lo;
      s_hi[threadIdx.x] = hi;
    }
    if (cb != cur_cb) {
#pragma unroll
      for (int k = 0; k < K; ++k) wk[k] = __ldg(reinterpret_cast<const unsigned long long*>(w + (size_t)k * d + c));
      bv = __ldg(reinterpret_cast<const unsigned long long*>(bias + c));
      cur_cb = cb;
    }
    const bool ok = mbar_wait(&full[st], (it / kDwStages) & 1, abort_flag);
    __syncthreads();  // s_lo / s_hi written; every thread's wait has returned
    if (__syncthreads_or(!ok)) break;
    const __half* tile = tiles + (size_t)st * HALO * 128;
#pragma unroll 1
    for (int grp = 0; grp < 2; ++grp) {
      const int j0 = rbase + grp * 8;
      const int lo = s_lo[j0], hi = s_hi[j0];
      const bool same = s_lo[j0 + 7] == lo;
      const int r = r0 + j0;
      float2 res[8];
      if (same && r - PAD >= lo && r + 7 + PAD < hi) {
        unsigned long long acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = bv;
#pragma unroll
        for (int t = 0; t < K + 7; ++t) {
          const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(tile + (j0 + t) * 128 + cc));
          const unsigned long long x = pk2(xf.x, xf.y);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int k = t - i;
            if (k >= 0 && k < K) acc[i] = fma2(wk[k], x, acc[i]);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 a = upk2(acc[i]);
          res[i] = make_float2(swish_t<__half>(a.x), swish_t<__half>(a.y));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) res[i] = make_float2(0.f, 0.f);
        int i0 = 0;
#pragma unroll 1
        while (i0 < 8) {
          const int li = s_lo[j0 + i0], hiI = s_hi[j0 + i0];
          int i1 = i0 + 1;
          while (i1 < 8 && s_lo[j0 + i1] == li) ++i1;
          const unsigned span = (unsigned)(hiI - li);
          unsigned long long a[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] = bv;
#pragma unroll
          for (int t = 0; t < K + 7; ++t) {
            unsigned long long x = 0ull;
            if ((unsigned)(r - PAD + t - li) < span) {
              const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(tile + (j0 + t) * 128 + cc));
              x = pk2(xf.x, xf.y);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int k = t - i;
              if (k >= 0 && k < K) a[i] = fma2(wk[k], x, a[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (i >= i0 && i < i1 && (unsigned)(r + i - li) < span) {
              const float2 q = upk2(a[i]);
              res[i] = make_float2(swish_t<__half>(q.x), swish_t<__half>(q.y));
            }
          i0 = i1;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (r + i >= rows) break;
        *reinterpret_cast<__half2*>(out + (size_t)(r + i) * d + c) = __floats2half2_rn(res[i].x, res[i].y);
      }
    }
    __syncthreads();  // stage st and s_lo / s_hi are free again
    if (threadIdx.x == 0) {
      fence_async_smem();
      issue(it + kDwStages);
    }
  }
  // loads still in flight (an early exit) land before the CTA leaves (bounded)
  if (threadIdx.x == 0) {
    for (int k = 0; k < kDwStages; ++k) {
      const int item = blockIdx.x + (it + k) * gridDim.x;
      if (item < n_items) mbar_settle(&full[(it + k) % kDwStages], ((it + k) / kDwStages) & 1, abort_flag, kWaitLimitNs);
    }
    if (s_abort) atomicExch(status, 1);
  }
}

// Any other odd kernel size (<= 63): one output per thread and tap loop.
template <typename T>
__global__ void __launch_bounds__(256)
dwconv_generic_kernel(const T* __restrict__ g, const float* __restrict__ w, const float* __restrict__ bias,
                      Clips clips, T* __restrict__ out, int rows, int d, int K) {
  const int pad = (K - 1) / 2;
  const size_t idx = (size_t)blockIdx.x * 256 + threadIdx.x;
  if (idx >= (size_t)rows * d) return;
  const int r = (int)(idx / d), c = (int)(idx % d);
  const int ci = clips.find(r, 1, 0);
  const int lo = clips.e(ci), hi = lo + clips.L2(ci);
  float a = 0.f;
  if (r >= lo && r < hi) {
    a = __ldg(bias + c);
    for (int k = 0; k < K; ++k) {
      const int src = r + k - pad;
      if (src >= lo && src < hi) a = fmaf(__ldg(w + (size_t)k * d + c), ld1(g + (size_t)src * d + c), a);
    }
    a = swish_t<T>(a);
  }
  if constexpr (sizeof(T) == 2) out[idx] = __float2half_rn(a);
  else out[idx] = a;
}

__global__ void scatter_kernel(const float* __restrict__ x, Clips clips, float* __restrict__ out, int t_max, int d) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= clips.B * t_max) return;
  const int b = row / t_max, t = row - b * t_max;
  float* o = out + (size_t)row * d;
  if (t < clips.L2(b)) {
    const float* xr = x + (size_t)(clips.e(b) + t) * d;
    for (int c = lane * 4; c < d; c += 128)
      *reinterpret_cast<float4*>(o + c) = *reinterpret_cast<const float4*>(xr + c);
  } else {
    for (int c = lane * 4; c < d; c += 128) *reinterpret_cast<float4*>(o + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// a ranks strictly above b in argmax order (NaN above everything, as in numpy)
__device__ __forceinline__ bool ranks_above(float a, float b) {
  if (isnan(b)) return false;
  return isnan(a) || a > b;
}

__global__ void logsoftmax_argmax_kernel(const float* __restrict__ logits, int ld, const int* __restrict__ lens,
                                         int batch, int t_max, int C, float* __restrict__ logp,
                                         int* __restrict__ argmax, const int* __restrict__ off) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= batch * t_max) return;
  const int b = row / t_max, t = row - b * t_max;
  if (t >= __ldg(lens + b)) {
    if (logp)
      for (int c = lane; c < C; c += 32) logp[(size_t)row * C + c] = 0.f;
    if (lane == 0) argmax[row] = -1;
    return;
  }
  const float* z = logits + (size_t)(off ? __ldg(off + b) + t : row) * ld;
  // First index of the maximum in the order of numpy's argmax: a NaN ranks above
  // every number (the first NaN wins) and a row of equal values, -inf included,
  // gives its first index.  A lane's own scan runs in increasing c and takes its
  // first element unconditionally; lanes without elements keep bi = INT_MAX.
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = lane; c < C; c += 32) {
    const float v = z[c];
    if (bi == 0x7fffffff || ranks_above(v, best)) { best = v; bi = c; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    const bool same = (ob == best) || (isnan(ob) && isnan(best));
    if (oi != 0x7fffffff && (bi == 0x7fffffff || ranks_above(ob, best) || (same && oi < bi))) { best = ob; bi = oi; }
  }
  float s = 0.f;
  for (int c = lane; c < C; c += 32) s += expf(z[c] - best);
  s = warp_sum(s);
  const float lse = best + logf(s);
  if (logp)
    for (int c = lane; c < C; c += 32) logp[(size_t)row * C + c] = z[c] - lse;
  if (lane == 0) argmax[row] = bi;
}

// One CTA (256 threads) per clip: keep_t = a_t != blank && (t == 0 || a_t != a_{t-1}),
// exclusive scan of keep flags over contiguous per-thread chunks, compaction.
__global__ void __launch_bounds__(256)
collapse_kernel(const int* __restrict__ argmax, const int* __restrict__ lens, int t_max, int blank,
                int* __restrict__ tokens, int* __restrict__ counts, int* __restrict__ frames) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int warp_tot[8];
  __shared__ int s_total;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int L = min(__ldg(lens + b), t_max);
  const int* a = argmax + (size_t)b * t_max;
  const int chunk = (L + 255) / 256;
  const int t0 = tid * chunk, t1 = min(t0 + chunk, L);
  int cnt = 0;
  for (int t = t0; t < t1; ++t) {
    const int v = a[t];
    cnt += (v != blank && (t == 0 || v != a[t - 1])) ? 1 : 0;
  }
  // inclusive warp scan
  int inc = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int i = 0; i < 8; ++i) { const int v = warp_tot[i]; warp_tot[i] = run; run += v; }
    s_total = run;
  }
  __syncthreads();
  int pos = warp_tot[w] + inc - cnt;
  int* tok = tokens + (size_t)b * t_max;
  int* frm = frames ? frames + (size_t)b * t_max : nullptr;
  for (int t = t0; t < t1; ++t) {
    const int v = a[t];
    if (v != blank && (t == 0 || v != a[t - 1])) {
      if (frm) frm[pos] = t;  // the first frame of the symbol's run
      tok[pos++] = v;
    }
  }
  const int total = s_total;
  for (int t = total + tid; t < t_max; t += 256) {
    tok[t] = -1;
    if (frm) frm[t] = -1;
  }
  if (tid == 0) counts[b] = total;
}

// One warp per valid frame v: find its clip b (largest b with off[b] <= v),
// read enc[b, v - off[b], :] and write the fp16 hi / lo split.
__global__ void split_hi_lo_kernel(const float* __restrict__ enc, const int* __restrict__ off, int batch, int t_max,
                                   int d, int rows, __half* __restrict__ a) {
  pdl_launch_dependents();
  pdl_wait();
  const int v = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (v >= rows) return;
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(off + mid) <= v) lo = mid; else hi = mid - 1;
  }
  const int t = v - __ldg(off + lo);
  const float* x = enc + ((size_t)lo * t_max + t) * d;
  __half* ah = a + (size_t)v * 2 * d;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 f = *reinterpret_cast<const float4*>(x + c);
    const __half2 h0 = __floats2half2_rn(f.x, f.y), h1 = __floats2half2_rn(f.z, f.w);
    const float2 b0 = __half22float2(h0), b1 = __half22float2(h1);
    const __half2 l0 = __floats2half2_rn(f.x - b0.x, f.y - b0.y), l1 = __floats2half2_rn(f.z - b1.x, f.w - b1.y);
    *reinterpret_cast<__half2*>(ah + c) = h0;
    *reinterpret_cast<__half2*>(ah + c + 2) = h1;
    *reinterpret_cast<__half2*>(ah + d + c) = l0;
    *reinterpret_cast<__half2*>(ah + d + c + 2) = l1;
  }
}

__global__ void f32_to_f16_kernel(const float* __restrict__ in, __half* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __float2half_rn(in[i]);
}

}  // namespace

#define GAM_NV_DISPATCH(d, CALL) \
  switch ((d) >> 7) {              \
    case 2: { constexpr int NV = 2; CALL; } break; \
    case 4: { constexpr int NV = 4; CALL; } break; \
    case 6: { constexpr int NV = 6; CALL; } break; \
    case 8: { constexpr int NV = 8; CALL; } break; \
    default: return cudaErrorInvalidValue; \
  }

// CTAs of 256 threads that fit on the device at once (per kernel, looked up once;
// a process drives one GPU model), capped by the 8-row groups there is work for.
template <auto KERNEL>
int resident_grid(int rows) {
  static const int resident = [] {
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, KERNEL, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
    return sms * per_sm;
  }();
  const int groups = (rows + 7) / 8;
  return groups < resident ? groups : resident;
}

template <typename T, int NV>
cudaError_t ln_t(const float* x, const float* g, const float* b, float eps, void* u, int rows, cudaStream_t s) {
  return launch_pdl(ln_kernel<T, NV>, resident_grid<ln_kernel<T, NV>>(rows), 256, 0, s, x, g, b, eps, (T*)u, rows);
}

cudaError_t launch_layernorm(const float* x, const float* g, const float* b, float eps, void* u, int u_half, int rows,
                             int d, cudaStream_t s) {
  if (d % 128 || d > 1024) return cudaErrorInvalidValue;
  if (rows <= 0) return cudaSuccess;
  if (u_half) GAM_NV_DISPATCH(d, return (ln_t<__half, NV>(x, g, b, eps, u, rows, s)))
  else GAM_NV_DISPATCH(d, return (ln_t<float, NV>(x, g, b, eps, u, rows, s)))
  return cudaErrorInvalidValue;
}

template <typename T, int NV>
cudaError_t ln_chain_t(float* x, const float* g1, const float* b1, const float* g2, const float* b2, float eps, void* u,
                       int rows, cudaStream_t s) {
  return launch_pdl(ln_chain_kernel<T, NV>, resident_grid<ln_chain_kernel<T, NV>>(rows), 256, 0, s, x, g1, b1, g2, b2,
                    eps, (T*)u, rows);
}

cudaError_t launch_layernorm_chain(float* x, const float* g1, const float* b1, const float* g2, const float* b2,
                                   float eps, void* u, int u_half, int rows, int d, cudaStream_t s) {
  if (d % 128 || d > 1024) return cudaErrorInvalidValue;
  if (rows <= 0) return cudaSuccess;
  if (u_half) GAM_NV_DISPATCH(d, return (ln_chain_t<__half, NV>(x, g1, b1, g2, b2, eps, u, rows, s)))
  else GAM_NV_DISPATCH(d, return (ln_chain_t<float, NV>(x, g1, b1, g2, b2, eps, u, rows, s)))
  return cudaErrorInvalidValue;
}

template <typename T, int DH, int NV>
cudaError_t rope_nv(const float* x, const float* g, const float* b, float eps, const float* cos_tab,
                    const float* sin_tab, Clips clips, void* u, void* urot, int rows, cudaStream_t s) {
  return launch_pdl(ln_rope_kernel<T, DH, NV>, resident_grid<ln_rope_kernel<T, DH, NV>>(rows), 256, 0, s, x, g, b, eps,
                    cos_tab, sin_tab, clips, (T*)u, (T*)urot, rows);
}

template <typename T, int DH>
cudaError_t rope_t(const float* x, const float* g, const float* b, float eps, const float* cos_tab,
                   const float* sin_tab, Clips clips, void* u, void* urot, int rows, int d, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  GAM_NV_DISPATCH(d, return (rope_nv<T, DH, NV>(x, g, b, eps, cos_tab, sin_tab, clips, u, urot, rows, s)))
  return cudaErrorInvalidValue;
}

cudaError_t launch_layernorm_rope(const float* x, const float* g, const float* b, float eps, const float* cos_tab,
                                  const float* sin_tab, Clips clips, void* u, void* urot, int u_half, int rows, int d,
                                  int d_head, cudaStream_t s) {
  if (d % 128 || d > 1024) return cudaErrorInvalidValue;
  if (d_head != 48 && d_head != 64) return cudaErrorInvalidValue;
  if (u_half) {
    if (d_head == 48) return rope_t<__half, 48>(x, g, b, eps, cos_tab, sin_tab, clips, u, urot, rows, d, s);
    return rope_t<__half, 64>(x, g, b, eps, cos_tab, sin_tab, clips, u, urot, rows, d, s);
  }
  if (d_head == 48) return rope_t<float, 48>(x, g, b, eps, cos_tab, sin_tab, clips, u, urot, rows, d, s);
  return rope_t<float, 64>(x, g, b, eps, cos_tab, sin_tab, clips, u, urot, rows, d, s);
}

template <int K>
cudaError_t dwconv_tma(const __half* g, const float* w, const float* bias, Clips clips, __half* out, int rows, int d,
                       int sm_count, int* status, cudaStream_t s) {
  constexpr int HALO = 64 + K - 1;
  CUtensorMap m;
  cudaError_t e = tma_map_2d(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g, (uint64_t)d, (uint64_t)rows, (uint64_t)d * 2, 128,
                             HALO, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  const int n_cb = d / 128, n_items = ((rows + 63) / 64) * n_cb;
  // two resident CTAs per SM; a multiple of n_cb, so that a CTA keeps one channel block
  int grid = std::min(n_items, 2 * sm_count);
  if (grid >= n_cb) grid -= grid % n_cb;
  const size_t smem = (size_t)kDwStages * HALO * 128 * 2 + 128;
  e = cudaFuncSetAttribute(dwconv_tma_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(dwconv_tma_kernel<K>, grid, 256, smem, s, m, w, bias, clips, out, rows, d, n_items, status);
}

template <typename T>
cudaError_t dwconv_t(const void* g, const float* w, const float* bias, Clips clips, void* out, int rows, int d, int K,
                     int sm_count, int* status, cudaStream_t s) {
  dim3 grid((rows + 63) / 64, d / 128);
  const T* gi = (const T*)g;
  T* o = (T*)out;
  if constexpr (sizeof(T) == 2) {  // fp16 activations: TMA-fed persistent form
    if (!status || (reinterpret_cast<uintptr_t>(g) & 15)) return cudaErrorInvalidValue;
    if (K == 31) return dwconv_tma<31>(gi, w, bias, clips, o, rows, d, sm_count, status, s);
    if (K == 5) return dwconv_tma<5>(gi, w, bias, clips, o, rows, d, sm_count, status, s);
    if (K == 15) return dwconv_tma<15>(gi, w, bias, clips, o, rows, d, sm_count, status, s);
  }
  if (K == 31) return launch_pdl(dwconv_kernel<T, 31>, grid, 256, 0, s, gi, w, bias, clips, o, rows, d);
  if (K == 5) return launch_pdl(dwconv_kernel<T, 5>, grid, 256, 0, s, gi, w, bias, clips, o, rows, d);
  if (K == 15) return launch_pdl(dwconv_kernel<T, 15>, grid, 256, 0, s, gi, w, bias, clips, o, rows, d);
  const size_t n = (size_t)rows * d;
  dwconv_generic_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(gi, w, bias, clips, o, rows, d, K);
  return cudaGetLastError();
}

cudaError_t launch_dwconv(const void* g, const float* w, const float* bias, Clips clips, void* out, int t_half,
                          int rows, int d, int K, int sm_count, int* status, cudaStream_t s) {
  if (d % 128 || K > 63 || (K & 1) == 0) return cudaErrorInvalidValue;
  if (t_half) return dwconv_t<__half>(g, w, bias, clips, out, rows, d, K, sm_count, status, s);
  return dwconv_t<float>(g, w, bias, clips, out, rows, d, K, sm_count, status, s);
}

cudaError_t launch_scatter_out(const float* x, Clips clips, float* out, int t_max, int d, cudaStream_t s) {
  const int rows = clips.B * t_max;
  return launch_pdl(scatter_kernel, (rows + 7) / 8, 256, 0, s, x, clips, out, t_max, d);
}

cudaError_t launch_logsoftmax_argmax(const float* logits, int ld, const int* lens, int batch, int t_max, int C,
                                     float* logp, int* argmax, cudaStream_t s, const int* off) {
  const int rows = batch * t_max;
  return launch_pdl(logsoftmax_argmax_kernel, (rows + 7) / 8, 256, 0, s, logits, ld, lens, batch, t_max, C, logp,
                    argmax, off);
}

cudaError_t launch_split_hi_lo(const float* enc, const int* off, int batch, int t_max, int d, int rows, __half* a,
                               cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (d % 128) return cudaErrorInvalidValue;
  return launch_pdl(split_hi_lo_kernel, (rows + 7) / 8, 256, 0, s, enc, off, batch, t_max, d, rows, a);
}

cudaError_t launch_collapse(const int* argmax, const int* lens, int batch, int t_max, int blank, int* tokens,
                            int* counts, cudaStream_t s, int* frames) {
  return launch_pdl(collapse_kernel, batch, 256, 0, s, argmax, lens, t_max, blank, tokens, counts, frames);
}

cudaError_t launch_f32_to_f16(const float* in, __half* out, int64_t n, cudaStream_t s) {
  f32_to_f16_kernel<<<148 * 8, 256, 0, s>>>(in, out, n);
  return cudaGetLastError();
}

}  // namespace gam
