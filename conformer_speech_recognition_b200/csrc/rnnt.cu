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

cudaError_t launch_rnnt_greedy(const float* eproj, const int* lens, const int* off, int batch, int t_max,
                               const float* gtab, const __half* whh, const __half* wp, const float* bp,
                               const __half* wo, const float* bo, int C, int P, int J, int max_symbols, int act,
                               int max_tokens, int* tokens, int* frames, int* counts, int* status, cudaStream_t s) {
  if (batch <= 0) return cudaSuccess;
  if (P % 8 || J % 8 || P < 8 || J < 8 || P > kMaxK || J > kMaxK || C < 2 || max_symbols < 1 || max_tokens < 1)
    return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(whh) | reinterpret_cast<uintptr_t>(wp) | reinterpret_cast<uintptr_t>(wo)) & 15)
    return cudaErrorInvalidValue;
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
