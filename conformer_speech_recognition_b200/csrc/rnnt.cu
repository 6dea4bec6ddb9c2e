// Greedy RNNT decoding on the GPU ("GigaAM on MLX: the transcripts matched, but
// the model was broken", "What we're porting": a single-layer LSTM of size 320
// plus a joint network; "GigaAM v3 RNNT -- MLX (Apple Silicon)": sequential
// greedy decode, LSTM bias = bias_ih + bias_hh, blank = len(vocabulary);
// "GigaAM v3 MLX", "Performance": the joint and the greedy loop dominate).
//
// The encoder half of the joint, W_enc f_t + b_enc, is one batched GEMM over
// all valid frames before this kernel runs (tensor cores, see the runtime).
// What is left is sequential per clip, so one CTA of 512 threads decodes one
// clip with its state in shared memory.  Each step is a few matrix-vector
// products against fp16 weights held in L2 (0.8 MB for W_hh, 0.2 MB for
// W_pred, C x 320 x 2 B for W_out).  A step waits on whole rows, so the rows
// stream through a ring of shared-memory chunks (32 rows each) with 1D TMA
// bulk copies: one thread keeps the next chunks in flight while the 16 warps
// take two rows of the landed chunk each (lanes read 16-byte pieces of a row,
// a warp reduction finishes the dot product) and release it:
//   predictor   (h, c) of the LSTM after the symbols emitted so far; the input
//               part of the gates, E[k] W_ih^T + b_ih + b_hh, is a table built
//               when the head is attached (row C: the zero start input), so a
//               step is gates = table[k] + W_hh h and the cell update;
//   pred proj   p = W_pred h + b_pred, once per predictor step;
//   joint       a = act(e_t + p), logits = W_out a + b_out, first-index argmax
//               (each warp over its rows in ascending order, then across warps);
//   loop        blank -> next frame; else store the symbol and its frame,
//               advance the predictor; at most max_symbols symbols per frame.
// fp32 state and accumulation.  The loop is bounded by T * (max_symbols + 1)
// decisions; every wait on the ring is bounded (a status word reports one that
// gave up, and the kernel then stops decoding that clip).
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "tc_common.cuh"

namespace gam {
namespace {

using namespace tc;

constexpr int kThreads = 512, kWarps = kThreads / 32;
constexpr int kRC = 2 * kWarps;          // rows per chunk: two per warp
constexpr int kMaxStages = 8;            // chunks in flight at most
constexpr int kMaxK = 1024;              // rows of at most 1024 fp16 weights
constexpr size_t kSmemBudget = 200 * 1024;

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 1D bulk copy global -> shared, completion counted on `bar` (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

struct RnntArgs {
  const float* eproj;    // [rows][J]: W_enc f + b_enc per valid frame
  const int* lens;       // [B] valid frames
  const int* off;        // [B] first eproj row of each clip (NULL: b * t_max)
  int t_max;
  const float* gtab;     // [(C + 1)][4P]
  const __half* whh;     // [4P][P]
  const __half* wp;      // [J][P]
  const float* bp;       // [J]
  const __half* wo;      // [C][J]
  const float* bo;       // [C]
  int C, P, J, max_symbols, act, max_tokens;
  int stages;            // ring stages of kRC * max(P, J) * 2 bytes
  int* tokens;           // [B][max_tokens]
  int* frames;           // [B][max_tokens] or NULL
  int* counts;           // [B]
  int* status;           // set when a bounded wait gave up
};

// The ring of weight chunks: stage s holds up to kRC rows; full[s] completes when
// its copy lands, empty[s] when all warps are done with it.  `seq` counts chunks
// over the whole kernel, so stage and phase follow from it.
struct Ring {
  uint8_t* buf;
  uint64_t* full;
  uint64_t* empty;
  uint32_t seq;
  uint32_t stage_bytes;  // kRC rows of the longest matrix row
  int stages;
  volatile int* abort_flag;
};

// Issue chunk c of a matrix (rows [c kRC, ...) of R rows, row_bytes each) into the
// stage of ring sequence number g, once that stage's previous chunk is released.
__device__ __forceinline__ bool issue_chunk(Ring& r, const uint8_t* W, int R, int row_bytes, int c, uint32_t g) {
  const uint32_t n = (uint32_t)r.stages;
  const int s = g % n;
  if (g >= n && !mbar_wait(&r.empty[s], ((g / n) - 1) & 1, r.abort_flag)) return false;
  const int rows = min(kRC, R - c * kRC);
  const uint32_t bytes = (uint32_t)rows * row_bytes;
  mbar_arrive_expect_tx(&r.full[s], bytes);
  bulk_load(r.buf + (size_t)s * r.stage_bytes, W + (size_t)c * kRC * row_bytes, bytes, &r.full[s]);
  return true;
}

// Streams the R x K fp16 matrix W (row-major) through the ring and hands each
// warp the dot products of its rows with x (shared memory, fp32): fn(row, dot)
// is called by lane 0 for every row, in ascending row order per warp.
template <class F>
__device__ __forceinline__ bool stream_rows(Ring& r, const __half* W, int R, int K, const float* x, F&& fn) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_bytes = K * 2, nch = (R + kRC - 1) / kRC;
  const uint8_t* Wb = reinterpret_cast<const uint8_t*>(W);
  bool ok = true;
  const uint32_t n = (uint32_t)r.stages;
  if (threadIdx.x == 0)
    for (int c = 0; c < min(nch, r.stages) && ok; ++c) ok = issue_chunk(r, Wb, R, row_bytes, c, r.seq + c);
  for (int c = 0; c < nch; ++c) {
    const uint32_t g = r.seq + c;
    const int s = g % n;
    if (!__all_sync(0xffffffffu, mbar_wait(&r.full[s], (g / n) & 1, r.abort_flag))) {
      ok = false;
      break;
    }
    const uint8_t* chunk = r.buf + (size_t)s * r.stage_bytes;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int rr = 2 * warp + i, row = c * kRC + rr;
      if (row < R) {
        const uint4* wrow = reinterpret_cast<const uint4*>(chunk + (size_t)rr * row_bytes);
        float acc = 0.f;
        for (int q = lane; q < K / 8; q += 32) {
          const uint4 w = wrow[q];
          const __half2* h = reinterpret_cast<const __half2*>(&w);
          const float4 x0 = *reinterpret_cast<const float4*>(x + 8 * q);
          const float4 x1 = *reinterpret_cast<const float4*>(x + 8 * q + 4);
          const float2 a = __half22float2(h[0]), b = __half22float2(h[1]), e = __half22float2(h[2]),
                       f = __half22float2(h[3]);
          acc = fmaf(a.x, x0.x, acc);
          acc = fmaf(a.y, x0.y, acc);
          acc = fmaf(b.x, x0.z, acc);
          acc = fmaf(b.y, x0.w, acc);
          acc = fmaf(e.x, x1.x, acc);
          acc = fmaf(e.y, x1.y, acc);
          acc = fmaf(f.x, x1.z, acc);
          acc = fmaf(f.y, x1.w, acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) fn(row, acc);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[s]);
    if (threadIdx.x == 0 && c + r.stages < nch && ok) ok = issue_chunk(r, Wb, R, row_bytes, c + r.stages, g + n);
  }
  r.seq += nch;
  return __syncthreads_and(ok) != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
rnnt_greedy_kernel(const RnntArgs p) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int P = p.P, J = p.J, C = p.C;
  const uint32_t stage_bytes = (uint32_t)kRC * max(P, J) * 2;
  uint8_t* ring_buf = smem_raw;
  float* h = reinterpret_cast<float*>(smem_raw + (size_t)p.stages * stage_bytes);  // [P]
  float* c = h + P;           // [P]
  float* gates = c + P;       // [4P]: W_hh h, before the table row is added
  float* pp = gates + 4 * P;  // [J]: W_pred h + b_pred
  float* a = pp + J;          // [J]: the joint's activation
  float* bps = a + J;         // [J]: b_pred
  float* logit = bps + J;     // [C]: W_out a, before b_out is added
  float* bos = logit + C;     // [C]: b_out
  __shared__ uint64_t s_full[kMaxStages], s_empty[kMaxStages];
  __shared__ float s_best[kWarps];
  __shared__ int s_bi[kWarps];
  constexpr int kNone = 0x7fffffff;
  __shared__ int s_k;
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kWarps);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  Ring ring{ring_buf, s_full, s_empty, 0u, stage_bytes, p.stages, reinterpret_cast<volatile int*>(&s_abort)};
  const int b = blockIdx.x;
  const int L = min(__ldg(p.lens + b), p.t_max);
  const size_t row0 = p.off ? (size_t)__ldg(p.off + b) : (size_t)b * p.t_max;
  const int blank = C - 1;

  for (int j = tid; j < P; j += kThreads) h[j] = c[j] = 0.f;
  for (int j = tid; j < J; j += kThreads) bps[j] = __ldg(p.bp + j);
  for (int j = tid; j < C; j += kThreads) bos[j] = __ldg(p.bo + j);
  __syncthreads();

  // one predictor step with input row `row` of the gate table, then the predictor projection
  auto lstm = [&](int row) {
    const float* gt = p.gtab + (size_t)row * 4 * P;
    if (!stream_rows(ring, p.whh, 4 * P, P, h, [&](int r, float d) { gates[r] = d; })) return false;
    for (int j = tid; j < P; j += kThreads) {
      const float ig = sigmoid_f(gates[j] + __ldg(gt + j)), fg = sigmoid_f(gates[P + j] + __ldg(gt + P + j));
      const float gg = tanhf(gates[2 * P + j] + __ldg(gt + 2 * P + j));
      const float og = sigmoid_f(gates[3 * P + j] + __ldg(gt + 3 * P + j));
      const float cn = fmaf(fg, c[j], ig * gg);
      c[j] = cn;
      h[j] = og * tanhf(cn);
    }
    __syncthreads();
    return stream_rows(ring, p.wp, J, P, h, [&](int r, float d) { pp[r] = d + bps[r]; });
  };

  bool ok = lstm(C);  // the start: zero input, zero state
  int count = 0;
  for (int t = 0; t < L && ok; ++t) {
    const float* e = p.eproj + (row0 + t) * J;
    for (int emitted = 0; emitted < p.max_symbols; ++emitted) {
      for (int j = tid; j < J; j += kThreads) {
        const float v = __ldg(e + j) + pp[j];
        a[j] = p.act == 0 ? fmaxf(v, 0.f) : tanhf(v);
      }
      __syncthreads();
      // logits over the streamed rows of W_out, then the first-index argmax: each
      // thread over its classes in ascending order, then across lanes and warps
      ok = stream_rows(ring, p.wo, C, J, a, [&](int r, float d) { logit[r] = d; });
      if (!ok) break;
      float best = -INFINITY;
      int bi = kNone;
      for (int r = tid; r < C; r += kThreads) {
        const float z = logit[r] + bos[r];
        if (bi == kNone || z > best) {
          best = z;
          bi = r;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != kNone && (bi == kNone || ob > best || (ob == best && oi < bi))) {
          best = ob;
          bi = oi;
        }
      }
      if (lane == 0) {
        s_best[warp] = best;
        s_bi[warp] = bi;
      }
      __syncthreads();
      if (tid == 0) {
        float bb = s_best[0];
        int k = s_bi[0];
        for (int w = 1; w < kWarps; ++w)
          if (s_bi[w] != kNone && (k == kNone || s_best[w] > bb || (s_best[w] == bb && s_bi[w] < k))) {
            bb = s_best[w];
            k = s_bi[w];
          }
        s_k = k;
        if (k != blank && count < p.max_tokens) {
          p.tokens[(size_t)b * p.max_tokens + count] = k;
          if (p.frames) p.frames[(size_t)b * p.max_tokens + count] = t;
        }
      }
      __syncthreads();
      const int k = s_k;
      if (k == blank) break;
      ++count;
      ok = lstm(k);
      if (!ok) break;
    }
  }
  // copies still in flight land before the CTA exits (bounded)
  if (tid == 0) {
    const uint32_t n = (uint32_t)p.stages;
    for (uint32_t g = ring.seq > n ? ring.seq - n : 0; g < ring.seq; ++g)
      mbar_settle(&s_full[g % n], (g / n) & 1, ring.abort_flag, kWaitLimitNs);
  }
  const int stored = min(count, p.max_tokens);
  for (int i = stored + tid; i < p.max_tokens; i += kThreads) {
    p.tokens[(size_t)b * p.max_tokens + i] = -1;
    if (p.frames) p.frames[(size_t)b * p.max_tokens + i] = -1;
  }
  if (tid == 0) {
    p.counts[b] = stored;
    if (s_abort) atomicExch(p.status, 1);
  }
}


// ---- weights resident in a cluster of CTAs (the default when they fit) ----
//
// A bulk copy into one SM delivers about 20 KB per half microsecond, so streaming
// the 1 MB of predictor weights through one SM costs tens of microseconds per
// emitted symbol.  Instead a cluster of kNC CTAs decodes one clip and each CTA
// keeps a slice of every matrix in its shared memory for the whole kernel:
//   CTA r   W_hh rows of the 4 gates for units [r P/kNC, (r+1) P/kNC), the
//           W_pred rows [r J/kNC, ...) and the W_out rows [r ceil(C/kNC), ...).
// A step exchanges only vectors through distributed shared memory:
//   LSTM    each CTA computes its units' gates, cell and hidden values and
//           writes its slice of h into every CTA (h is double-buffered);
//           cluster barrier;
//   pred    each CTA computes its slice of p = W_pred h + b_pred and writes it
//           into every CTA; cluster barrier;
//   joint   each CTA forms a = act(e_t + p) in full, the logits of its classes
//           and their first-index maximum, and writes (max, index) into every
//           CTA's slot (double-buffered by decision); cluster barrier; every CTA
//           then reduces the kNC candidates in rank order, so all take the same
//           decision and the control flow stays uniform across the cluster.
// Dot products: 8 lanes per row (16-byte loads, 3 shuffles), 4 rows per warp.
// The barriers are hardware cluster barriers, which every CTA reaches in the
// same order; there is no spin-wait.
constexpr int kNC = 8;
constexpr int kCThreads = 512, kCWarps = kCThreads / 32;
constexpr size_t kClusterSmemMax = 226 * 1024;  // beside the static shared memory

struct ClusterArgs {
  const float* eproj;
  const int* lens;
  const int* off;
  const int* order;      // [B]: clip decoded by cluster i (longest first)
  int t_max;
  const float* gtab;
  const __half* whh;
  const __half* wp;
  const float* bp;
  const __half* wo;
  const float* bo;
  int C, P, J, max_symbols, act, max_tokens;
  int* tokens;
  int* frames;
  int* counts;
};

struct ClusterLayout {
  int Pu, Ju, Cu;
  size_t whh, wp, wo, h, cst, graw, pp, a, e, bps, bos, logit, slots, total;
};

__host__ __device__ inline ClusterLayout cluster_layout(int C, int P, int J) {
  ClusterLayout L;
  L.Pu = P / kNC;
  L.Ju = J / kNC;
  L.Cu = (C + kNC - 1) / kNC;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += (bytes + 15) & ~(size_t)15;
    return at;
  };
  L.whh = take((size_t)4 * L.Pu * P * 2);
  L.wp = take((size_t)L.Ju * P * 2);
  L.wo = take((size_t)L.Cu * J * 2);
  L.h = take((size_t)2 * P * 4);
  L.cst = take((size_t)L.Pu * 4);
  L.graw = take((size_t)4 * L.Pu * 4);
  L.pp = take((size_t)J * 4);
  L.a = take((size_t)J * 4);
  L.e = take((size_t)J * 4);
  L.bps = take((size_t)L.Ju * 4);
  L.bos = take((size_t)L.Cu * 4);
  L.logit = take((size_t)L.Cu * 4);
  L.slots = take((size_t)2 * kNC * 8);  // [2][kNC] of (float max, int index)
  L.total = o;
  return L;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_peer_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_peer_s32(uint32_t addr, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Write v into location `local` of every CTA of the cluster (this one included).
__device__ __forceinline__ void broadcast_f32(float* local, float v) {
#pragma unroll
  for (int r = 0; r < kNC; ++r) st_peer_f32(peer_addr(local, r), v);
}

// fn(row, dot) for the rows [0, R) of the K-column fp16 matrix W (shared memory,
// row-major) against x (shared memory, fp32): 8 lanes per row, called by the
// row's first lane.
template <class F>
__device__ __forceinline__ void smem_dots(const __half* W, int R, int K, const float* x, F&& fn) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, l8 = lane & 7, nq = K / 8;
  for (int base = warp * 4; base < R; base += kCWarps * 4) {
    const int row = base + g;
    float acc = 0.f;
    if (row < R) {
      const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)row * K);
      for (int q = l8; q < nq; q += 8) {
        const uint4 w = wr[q];
        const __half2* hh = reinterpret_cast<const __half2*>(&w);
        const float4 x0 = *reinterpret_cast<const float4*>(x + 8 * q);
        const float4 x1 = *reinterpret_cast<const float4*>(x + 8 * q + 4);
        const float2 p0 = __half22float2(hh[0]), p1 = __half22float2(hh[1]), p2 = __half22float2(hh[2]),
                     p3 = __half22float2(hh[3]);
        acc = fmaf(p0.x, x0.x, acc);
        acc = fmaf(p0.y, x0.y, acc);
        acc = fmaf(p1.x, x0.z, acc);
        acc = fmaf(p1.y, x0.w, acc);
        acc = fmaf(p2.x, x1.x, acc);
        acc = fmaf(p2.y, x1.y, acc);
        acc = fmaf(p3.x, x1.z, acc);
        acc = fmaf(p3.y, x1.w, acc);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (row < R && l8 == 0) fn(row, acc);
  }
}

// Copy `bytes` (a multiple of 16) from global to shared memory with all threads.
__device__ __forceinline__ void copy16(void* dst, const void* src, size_t bytes) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  const uint4* s = reinterpret_cast<const uint4*>(src);
  for (size_t i = threadIdx.x; i < bytes / 16; i += kCThreads) d[i] = __ldg(s + i);
}

__global__ void __launch_bounds__(kCThreads, 1) rnnt_cluster_kernel(const ClusterArgs p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int C = p.C, P = p.P, J = p.J;
  const ClusterLayout Ly = cluster_layout(C, P, J);
  const int Pu = Ly.Pu, Ju = Ly.Ju, Cu = Ly.Cu;
  __half* whh = reinterpret_cast<__half*>(smem_raw + Ly.whh);  // [4 Pu][P]: gate g, unit i at row g Pu + i
  __half* wp = reinterpret_cast<__half*>(smem_raw + Ly.wp);    // [Ju][P]
  __half* wo = reinterpret_cast<__half*>(smem_raw + Ly.wo);    // [Cu][J]
  float* hbuf = reinterpret_cast<float*>(smem_raw + Ly.h);     // [2][P]
  float* cst = reinterpret_cast<float*>(smem_raw + Ly.cst);    // [Pu]
  float* graw = reinterpret_cast<float*>(smem_raw + Ly.graw);  // [4 Pu]
  float* pp = reinterpret_cast<float*>(smem_raw + Ly.pp);      // [J]: W_pred h + b_pred
  float* a = reinterpret_cast<float*>(smem_raw + Ly.a);        // [J]
  float* e = reinterpret_cast<float*>(smem_raw + Ly.e);        // [J]: W_enc f_t + b_enc
  float* bps = reinterpret_cast<float*>(smem_raw + Ly.bps);    // [Ju]
  float* bos = reinterpret_cast<float*>(smem_raw + Ly.bos);    // [Cu]
  float* logit = reinterpret_cast<float*>(smem_raw + Ly.logit);
  float* slot_v = reinterpret_cast<float*>(smem_raw + Ly.slots);  // [2][kNC]
  int* slot_i = reinterpret_cast<int*>(slot_v + 2 * kNC);          // [2][kNC]
  __shared__ float s_best[kCWarps];
  __shared__ int s_bi[kCWarps];
  constexpr int kNone = 0x7fffffff;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)cluster_rank();
  const int b = __ldg(p.order + blockIdx.x / kNC);
  const int L = min(__ldg(p.lens + b), p.t_max);
  const size_t row0 = p.off ? (size_t)__ldg(p.off + b) : (size_t)b * p.t_max;
  const int blank = C - 1;
  const int u0 = rank * Pu, j0 = rank * Ju, c0 = rank * Cu;
  const int Cn = max(0, min(Cu, C - c0));

  // this CTA's weight slices, resident for the whole kernel
  for (int g = 0; g < 4; ++g)
    copy16(whh + (size_t)g * Pu * P, p.whh + ((size_t)g * P + u0) * P, (size_t)Pu * P * 2);
  copy16(wp, p.wp + (size_t)j0 * P, (size_t)Ju * P * 2);
  if (Cn > 0) copy16(wo, p.wo + (size_t)c0 * J, (size_t)Cn * J * 2);
  for (int j = tid; j < Ju; j += kCThreads) bps[j] = __ldg(p.bp + j0 + j);
  for (int j = tid; j < Cn; j += kCThreads) bos[j] = __ldg(p.bo + c0 + j);
  for (int j = tid; j < 2 * P; j += kCThreads) hbuf[j] = 0.f;
  for (int j = tid; j < Pu; j += kCThreads) cst[j] = 0.f;
  cluster_sync_all();  // every CTA of the cluster runs, and its state is initialised

  int hb = 0;  // h buffer holding the current hidden state
  // one predictor step with input row `row` of the gate table, then the predictor projection
  auto lstm = [&](int row) {
    float gt0 = 0.f, gt1 = 0.f, gt2 = 0.f, gt3 = 0.f;
    if (tid < Pu) {  // the table entries of this thread's unit, loaded ahead of the dot products
      const float* gr = p.gtab + (size_t)row * 4 * P + u0 + tid;
      gt0 = __ldg(gr);
      gt1 = __ldg(gr + P);
      gt2 = __ldg(gr + 2 * P);
      gt3 = __ldg(gr + 3 * P);
    }
    smem_dots(whh, 4 * Pu, P, hbuf + hb * P, [&](int r, float d) { graw[r] = d; });
    __syncthreads();
    if (tid < Pu) {
      const float ig = sigmoid_f(graw[tid] + gt0), fg = sigmoid_f(graw[Pu + tid] + gt1);
      const float gg = tanhf(graw[2 * Pu + tid] + gt2), og = sigmoid_f(graw[3 * Pu + tid] + gt3);
      const float cn = fmaf(fg, cst[tid], ig * gg);
      cst[tid] = cn;
      broadcast_f32(hbuf + (hb ^ 1) * P + u0 + tid, og * tanhf(cn));
    }
    cluster_sync_all();
    hb ^= 1;
    smem_dots(wp, Ju, P, hbuf + hb * P, [&](int r, float d) { broadcast_f32(pp + j0 + r, d + bps[r]); });
    cluster_sync_all();
  };

  lstm(C);  // the start: zero input, zero state
  int count = 0, par = 0;
  float e_next = (tid < J && L > 0) ? __ldg(p.eproj + row0 * J + tid) : 0.f;
  for (int t = 0; t < L; ++t) {
    if (tid < J) e[tid] = e_next;
    if (tid < J && t + 1 < L) e_next = __ldg(p.eproj + (row0 + t + 1) * J + tid);  // next frame, ahead
    for (int emitted = 0; emitted < p.max_symbols; ++emitted) {
      __syncthreads();
      for (int j = tid; j < J; j += kCThreads) {
        const float v = e[j] + pp[j];
        a[j] = p.act == 0 ? fmaxf(v, 0.f) : tanhf(v);
      }
      __syncthreads();
      smem_dots(wo, Cn, J, a, [&](int r, float d) { logit[r] = d; });
      __syncthreads();
      // first-index maximum over this CTA's classes (ascending per thread, then lanes, warps)
      float best = -INFINITY;
      int bi = kNone;
      for (int r = tid; r < Cn; r += kCThreads) {
        const float z = logit[r] + bos[r];
        if (bi == kNone || z > best) {
          best = z;
          bi = c0 + r;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != kNone && (bi == kNone || ob > best || (ob == best && oi < bi))) {
          best = ob;
          bi = oi;
        }
      }
      if (lane == 0) {
        s_best[warp] = best;
        s_bi[warp] = bi;
      }
      __syncthreads();
      if (tid < kNC) {  // thread r sends this CTA's candidate to CTA r
        float bb = s_best[0];
        int k = s_bi[0];
        for (int w = 1; w < kCWarps; ++w)
          if (s_bi[w] != kNone && (k == kNone || s_best[w] > bb || (s_best[w] == bb && s_bi[w] < k))) {
            bb = s_best[w];
            k = s_bi[w];
          }
        st_peer_f32(peer_addr(slot_v + par * kNC + rank, tid), bb);
        st_peer_s32(peer_addr(slot_i + par * kNC + rank, tid), k);
      }
      cluster_sync_all();
      // the same reduction in every CTA: candidates in rank order cover ascending class ranges
      float bb = slot_v[par * kNC];
      int k = slot_i[par * kNC];
      for (int r = 1; r < kNC; ++r) {
        const int ki = slot_i[par * kNC + r];
        const float vi = slot_v[par * kNC + r];
        if (ki != kNone && (k == kNone || vi > bb)) {
          bb = vi;
          k = ki;
        }
      }
      par ^= 1;
      if (k == blank || k == kNone) break;
      if (rank == 0 && tid == 0 && count < p.max_tokens) {
        p.tokens[(size_t)b * p.max_tokens + count] = k;
        if (p.frames) p.frames[(size_t)b * p.max_tokens + count] = t;
      }
      ++count;
      lstm(k);
    }
  }
  if (rank == 0) {
    const int stored = min(count, p.max_tokens);
    for (int i = stored + tid; i < p.max_tokens; i += kCThreads) {
      p.tokens[(size_t)b * p.max_tokens + i] = -1;
      if (p.frames) p.frames[(size_t)b * p.max_tokens + i] = -1;
    }
    if (tid == 0) p.counts[b] = stored;
  }
  cluster_sync_all();  // no CTA leaves while another may still write into its shared memory
}

}  // namespace

size_t rnnt_state_bytes(int C, int P, int J) { return sizeof(float) * ((size_t)6 * P + 3 * (size_t)J + 2 * (size_t)C); }

// Ring stages that fit the shared-memory budget beside the state vectors (0: none fit).
int rnnt_stages(int C, int P, int J) {
  const size_t state = rnnt_state_bytes(C, P, J);
  const size_t stage = (size_t)kRC * std::max(P, J) * 2;
  if (state >= kSmemBudget) return 0;
  return (int)std::min<size_t>(kMaxStages, (kSmemBudget - state) / stage);
}

// Dynamic shared memory of the decode kernel; SIZE_MAX when fewer than two ring stages fit.
size_t rnnt_smem_bytes(int C, int P, int J) {
  const int st = rnnt_stages(C, P, J);
  if (st < 2) return SIZE_MAX;
  return (size_t)st * kRC * std::max(P, J) * 2 + rnnt_state_bytes(C, P, J);
}

// The cluster form needs its slices and vectors in shared memory, J <= one value per
// thread, and a cluster of kNC such CTAs that the GPU can hold at once.
bool rnnt_cluster_fits(int C, int P, int J) {
  if (P % kNC || J % kNC || J > kCThreads) return false;
  const size_t smem = cluster_layout(C, P, J).total;
  if (smem > kClusterSmemMax) return false;
  static int cached_smem = -1, cached_ok = 0;
  if (cached_smem == (int)smem) return cached_ok != 0;
  int n = 0;
  if (cudaFuncSetAttribute(rnnt_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kNC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(kNC);
    cfg.blockDim = dim3(kCThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, rnnt_cluster_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached_smem = (int)smem;
  cached_ok = n > 0;
  return n > 0;
}

// GAM_RNNT=ring selects the streaming form for every head (read at each launch).
bool rnnt_force_ring() {
  const char* e = std::getenv("GAM_RNNT");
  return e && std::strcmp(e, "ring") == 0;
}

cudaError_t launch_rnnt_greedy(const float* eproj, const int* lens, const int* off, const int* order, int batch,
                               int t_max, const float* gtab, const __half* whh, const __half* wp, const float* bp,
                               const __half* wo, const float* bo, int C, int P, int J, int max_symbols, int act,
                               int max_tokens, int* tokens, int* frames, int* counts, int* status, cudaStream_t s) {
  if (batch <= 0) return cudaSuccess;
  if (P % 8 || J % 8 || P < 8 || J < 8 || P > kMaxK || J > kMaxK || C < 2 || max_symbols < 1 || max_tokens < 1)
    return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(whh) | reinterpret_cast<uintptr_t>(wp) | reinterpret_cast<uintptr_t>(wo)) & 15)
    return cudaErrorInvalidValue;
  if (order && !rnnt_force_ring() && rnnt_cluster_fits(C, P, J)) {
    ClusterArgs c;
    c.eproj = eproj;
    c.lens = lens;
    c.off = off;
    c.order = order;
    c.t_max = t_max;
    c.gtab = gtab;
    c.whh = whh;
    c.wp = wp;
    c.bp = bp;
    c.wo = wo;
    c.bo = bo;
    c.C = C;
    c.P = P;
    c.J = J;
    c.max_symbols = max_symbols;
    c.act = act;
    c.max_tokens = max_tokens;
    c.tokens = tokens;
    c.frames = frames;
    c.counts = counts;
    const size_t smem = cluster_layout(C, P, J).total;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kNC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kNC * batch);
    cfg.blockDim = dim3(kCThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rnnt_cluster_kernel, c);
  }
  RnntArgs a;
  a.eproj = eproj;
  a.lens = lens;
  a.off = off;
  a.t_max = t_max;
  a.gtab = gtab;
  a.whh = whh;
  a.wp = wp;
  a.bp = bp;
  a.wo = wo;
  a.bo = bo;
  a.C = C;
  a.P = P;
  a.J = J;
  a.max_symbols = max_symbols;
  a.act = act;
  a.max_tokens = max_tokens;
  a.tokens = tokens;
  a.frames = frames;
  a.counts = counts;
  a.status = status;
  a.stages = rnnt_stages(C, P, J);
  if (a.stages < 2) return cudaErrorInvalidValue;  // n_classes too large for the state in shared memory
  const size_t smem = rnnt_smem_bytes(C, P, J);
  cudaError_t e = cudaFuncSetAttribute(rnnt_greedy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(rnnt_greedy_kernel, batch, kThreads, smem, s, a);
}

}  // namespace gam
