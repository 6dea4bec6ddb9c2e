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
// products against fp16 weights that stay in L2 (0.8 MB for W_hh, 0.2 MB for
// W_pred, C x 320 x 2 B for W_out): a warp takes whole rows, each lane reads
// 16-byte chunks of the row (8 weights) and the matching fp32 inputs from
// shared memory, a warp reduction finishes the dot product, and every warp
// keeps several rows' loads in flight, since the step is bound by L2 latency:
//   predictor   (h, c) of the LSTM after the symbols emitted so far; the input
//               part of the gates, E[k] W_ih^T + b_ih + b_hh, is a table built
//               when the head is attached (row C: the zero start input), so a
//               step is gates = table[k] + W_hh h and the cell update;
//   pred proj   p = W_pred h + b_pred, once per predictor step;
//   joint       a = act(e_t + p), logits = W_out a + b_out, first-index argmax
//               (per warp over its rows, then across warps);
//   loop        blank -> next frame; else store the symbol and its frame,
//               advance the predictor; at most max_symbols symbols per frame.
// fp32 state and accumulation.  The loop is bounded by T * (max_symbols + 1)
// decisions; there are no waits.
#include "common.cuh"

namespace gam {
namespace {

constexpr int kThreads = 512, kWarps = kThreads / 32;
constexpr int kRowsInFlight = 4;  // rows per warp whose loads are issued together

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// dot(W[row, 0:K], x) for K % 8 == 0, rows of W 16-byte aligned (row stride K
// halves), x in shared memory; every lane of the warp returns the sum.
template <int NR>
__device__ __forceinline__ void warp_dots(const __half* __restrict__ W, int K, const int (&rows)[NR],
                                          const float* x, float (&out)[NR]) {
  const int lane = threadIdx.x & 31;
  float acc[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) acc[i] = 0.f;
  for (int c = lane; c < K / 8; c += 32) {
    uint4 w[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i)
      w[i] = rows[i] >= 0 ? __ldg(reinterpret_cast<const uint4*>(W + (size_t)rows[i] * K) + c) : make_uint4(0, 0, 0, 0);
    const float4 x0 = *reinterpret_cast<const float4*>(x + 8 * c);
    const float4 x1 = *reinterpret_cast<const float4*>(x + 8 * c + 4);
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const __half2* h = reinterpret_cast<const __half2*>(&w[i]);
      const float2 a = __half22float2(h[0]), b = __half22float2(h[1]), e = __half22float2(h[2]),
                   f = __half22float2(h[3]);
      float s = acc[i];
      s = fmaf(a.x, x0.x, s);
      s = fmaf(a.y, x0.y, s);
      s = fmaf(b.x, x0.z, s);
      s = fmaf(b.y, x0.w, s);
      s = fmaf(e.x, x1.x, s);
      s = fmaf(e.y, x1.y, s);
      s = fmaf(f.x, x1.z, s);
      s = fmaf(f.y, x1.w, s);
      acc[i] = s;
    }
  }
#pragma unroll
  for (int i = 0; i < NR; ++i) out[i] = warp_sum(acc[i]);
}

// y[r] = bias[r] + dot(W[r], x) for r < R, rows spread over the warps.
__device__ __forceinline__ void matvec(const __half* __restrict__ W, const float* __restrict__ bias, int R, int K,
                                       const float* x, float* y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r0 = warp * kRowsInFlight; r0 < R; r0 += kWarps * kRowsInFlight) {
    int rows[kRowsInFlight];
#pragma unroll
    for (int i = 0; i < kRowsInFlight; ++i) rows[i] = r0 + i < R ? r0 + i : -1;
    float d[kRowsInFlight];
    warp_dots<kRowsInFlight>(W, K, rows, x, d);
    if (lane < kRowsInFlight && rows[lane] >= 0) {
      float v = d[0];
#pragma unroll
      for (int i = 1; i < kRowsInFlight; ++i)
        if (lane == i) v = d[i];
      y[rows[lane]] = v + __ldg(bias + rows[lane]);
    }
  }
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
  int* tokens;           // [B][max_tokens]
  int* frames;           // [B][max_tokens] or NULL
  int* counts;           // [B]
};

__global__ void __launch_bounds__(kThreads)
rnnt_greedy_kernel(const RnntArgs p) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) float sm[];
  const int P = p.P, J = p.J, C = p.C;
  float* h = sm;              // [P]
  float* c = h + P;           // [P]
  float* gates = c + P;       // [4P]
  float* pp = gates + 4 * P;  // [J]
  float* a = pp + J;          // [J]
  __shared__ float s_best[kWarps];
  __shared__ int s_bi[kWarps];
  __shared__ int s_k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x;
  const int L = min(__ldg(p.lens + b), p.t_max);
  const size_t row0 = p.off ? (size_t)__ldg(p.off + b) : (size_t)b * p.t_max;
  const int blank = C - 1;

  for (int j = tid; j < P; j += kThreads) h[j] = c[j] = 0.f;
  __syncthreads();

  // one predictor step with input row `row` of the gate table: (h, c) <- LSTM(x_row, (h, c)),
  // then the predictor projection of the new h
  auto lstm = [&](int row) {
    matvec(p.whh, p.gtab + (size_t)row * 4 * P, 4 * P, P, h, gates);
    __syncthreads();
    for (int j = tid; j < P; j += kThreads) {
      const float ig = sigmoid_f(gates[j]), fg = sigmoid_f(gates[P + j]);
      const float gg = tanhf(gates[2 * P + j]), og = sigmoid_f(gates[3 * P + j]);
      const float cn = fmaf(fg, c[j], ig * gg);
      c[j] = cn;
      h[j] = og * tanhf(cn);
    }
    __syncthreads();
    matvec(p.wp, p.bp, J, P, h, pp);
    __syncthreads();
  };

  lstm(C);  // the start: zero input, zero state
  int count = 0;
  for (int t = 0; t < L; ++t) {
    const float* e = p.eproj + (row0 + t) * J;
    for (int emitted = 0; emitted < p.max_symbols; ++emitted) {
      for (int j = tid; j < J; j += kThreads) {
        const float v = __ldg(e + j) + pp[j];
        a[j] = p.act == 0 ? fmaxf(v, 0.f) : tanhf(v);
      }
      __syncthreads();
      // logits row by row over the warps; each warp keeps its first-index maximum
      float best = -INFINITY;
      int bi = 0x7fffffff;
      for (int r0 = warp * kRowsInFlight; r0 < C; r0 += kWarps * kRowsInFlight) {
        int rows[kRowsInFlight];
#pragma unroll
        for (int i = 0; i < kRowsInFlight; ++i) rows[i] = r0 + i < C ? r0 + i : -1;
        float d[kRowsInFlight];
        warp_dots<kRowsInFlight>(p.wo, J, rows, a, d);
#pragma unroll
        for (int i = 0; i < kRowsInFlight; ++i)
          if (rows[i] >= 0) {
            const float z = d[i] + __ldg(p.bo + rows[i]);
            if (bi == 0x7fffffff || z > best) { best = z; bi = rows[i]; }  // rows ascend within a warp
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
          if (s_bi[w] != 0x7fffffff && (k == 0x7fffffff || s_best[w] > bb || (s_best[w] == bb && s_bi[w] < k))) {
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
      lstm(k);
    }
  }
  const int stored = min(count, p.max_tokens);
  for (int i = stored + tid; i < p.max_tokens; i += kThreads) {
    p.tokens[(size_t)b * p.max_tokens + i] = -1;
    if (p.frames) p.frames[(size_t)b * p.max_tokens + i] = -1;
  }
  if (tid == 0) p.counts[b] = stored;
}

}  // namespace

size_t rnnt_smem_bytes(int C, int P, int J) {
  (void)C;
  return sizeof(float) * ((size_t)6 * P + 2 * J);
}

cudaError_t launch_rnnt_greedy(const float* eproj, const int* lens, const int* off, int batch, int t_max,
                               const float* gtab, const __half* whh, const __half* wp, const float* bp,
                               const __half* wo, const float* bo, int C, int P, int J, int max_symbols, int act,
                               int max_tokens, int* tokens, int* frames, int* counts, cudaStream_t s) {
  if (batch <= 0) return cudaSuccess;
  if (P % 8 || J % 8 || C < 2 || max_symbols < 1 || max_tokens < 1) return cudaErrorInvalidValue;
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
  const size_t smem = rnnt_smem_bytes(C, P, J);
  cudaError_t e = cudaFuncSetAttribute(rnnt_greedy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(rnnt_greedy_kernel, batch, kThreads, smem, s, a);
}

}  // namespace gam
