// Greedy RNNT decoding on the GPU ("GigaAM on MLX: the transcripts matched, but
// the model was broken", "What we're porting": a single-layer LSTM of size 320
// plus a joint network; "GigaAM v3 RNNT -- MLX (Apple Silicon)": sequential
// greedy decode, LSTM bias = bias_ih + bias_hh, blank = len(vocabulary);
// "GigaAM v3 MLX", "Performance": the joint and the greedy loop dominate).
//
// The encoder half of the joint, W_enc f_t + b_enc, is one batched GEMM over
// all valid frames before this kernel runs (tensor cores, see the runtime).
// What is left is sequential per clip, so one CTA of 256 threads decodes one
// clip with its state in shared memory:
//   predictor   (h, c) of the LSTM after the symbols emitted so far; the input
//               part of the gates, E[k] W_ih^T + b_ih + b_hh, is a table built
//               when the head is attached (row C: the zero start input), so a
//               step is gates = table[k] + W_hh h (thread per pair of gate rows,
//               W_hh^T read as half2 along the rows) and the cell update;
//   pred proj   p = W_pred h + b_pred, once per predictor step;
//   joint       a = act(e_t + p), logits = W_out a + b_out (the classes split
//               over the threads, each class's dot product over a slice of the
//               joint width when there are few classes), first-index argmax;
//   loop        blank -> next frame; else store the symbol and its frame,
//               advance the predictor; at most max_symbols symbols per frame.
// fp32 state and accumulation, fp16 weights read through L2.  The loop is
// bounded by T * (max_symbols + 1) decisions; there are no waits.
#include "common.cuh"

namespace gam {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

struct RnntArgs {
  const float* eproj;    // [rows][J]: W_enc f + b_enc per valid frame
  const int* lens;       // [B] valid frames
  const int* off;        // [B] first eproj row of each clip (NULL: b * t_max)
  int t_max;
  const float* gtab;     // [(C + 1)][4P]
  const __half2* whhT;   // [P][2P] half2 pairs of gate rows (row pair q = rows 2q, 2q + 1)
  const __half2* wpT;    // [P][J / 2]
  const float* bp;       // [J]
  const __half* woT;     // [J][C]
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
  extern __shared__ float sm[];
  const int P = p.P, J = p.J, C = p.C;
  float* h = sm;              // [P]
  float* c = h + P;           // [P]
  float* gates = c + P;       // [4P]
  float* pp = gates + 4 * P;  // [J]
  float* a = pp + J;          // [J]
  float* zp = a + J;          // [max(C, kThreads)] partial logits
  __shared__ float s_best[kThreads / 32];
  __shared__ int s_bi[kThreads / 32];
  __shared__ int s_k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x;
  const int L = min(__ldg(p.lens + b), p.t_max);
  const size_t row0 = p.off ? (size_t)__ldg(p.off + b) : (size_t)b * p.t_max;
  const int blank = C - 1;
  // classes split: nparts slices of the joint width per class when C < threads
  const int nparts = C < kThreads ? kThreads / C : 1;
  const int jlen = (J + nparts - 1) / nparts;

  for (int j = tid; j < P; j += kThreads) h[j] = c[j] = 0.f;
  __syncthreads();

  // one predictor step with input row `row` of the gate table: (h, c) <- LSTM(x_row, (h, c))
  auto lstm = [&](int row) {
    const float* gt = p.gtab + (size_t)row * 4 * P;
    for (int q = tid; q < 2 * P; q += kThreads) {  // gate rows 2q, 2q + 1
      float s0 = __ldg(gt + 2 * q), s1 = __ldg(gt + 2 * q + 1);
      for (int k = 0; k < P; ++k) {
        const float2 w = __half22float2(p.whhT[(size_t)k * 2 * P + q]);
        const float hk = h[k];
        s0 = fmaf(w.x, hk, s0);
        s1 = fmaf(w.y, hk, s1);
      }
      gates[2 * q] = s0;
      gates[2 * q + 1] = s1;
    }
    __syncthreads();
    for (int j = tid; j < P; j += kThreads) {
      const float ig = sigmoid_f(gates[j]), fg = sigmoid_f(gates[P + j]);
      const float gg = tanhf(gates[2 * P + j]), og = sigmoid_f(gates[3 * P + j]);
      const float cn = fmaf(fg, c[j], ig * gg);
      c[j] = cn;
      h[j] = og * tanhf(cn);
    }
    __syncthreads();
    for (int q = tid; q < J / 2; q += kThreads) {  // pred projection, two outputs per thread
      float s0 = __ldg(p.bp + 2 * q), s1 = __ldg(p.bp + 2 * q + 1);
      for (int k = 0; k < P; ++k) {
        const float2 w = __half22float2(p.wpT[(size_t)k * (J / 2) + q]);
        s0 = fmaf(w.x, h[k], s0);
        s1 = fmaf(w.y, h[k], s1);
      }
      pp[2 * q] = s0;
      pp[2 * q + 1] = s1;
    }
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
      // logits: partial dot products over slices of the joint width
      if (nparts > 1) {
        if (tid < nparts * C) {
          const int cls = tid % C, part = tid / C;
          const int j0 = part * jlen, j1 = min(J, j0 + jlen);
          float s = 0.f;
          for (int j = j0; j < j1; ++j) s = fmaf(__half2float(p.woT[(size_t)j * C + cls]), a[j], s);
          zp[part * C + cls] = s;
        }
      } else {
        for (int cls = tid; cls < C; cls += kThreads) {
          float s = 0.f;
          for (int j = 0; j < J; ++j) s = fmaf(__half2float(p.woT[(size_t)j * C + cls]), a[j], s);
          zp[cls] = s;
        }
      }
      __syncthreads();
      // first-index argmax of bias + partial sums
      float best = -INFINITY;
      int bi = 0x7fffffff;
      for (int cls = tid; cls < C; cls += kThreads) {
        float z = __ldg(p.bo + cls);
        for (int part = 0; part < nparts; ++part) z += zp[part * C + cls];
        if (bi == 0x7fffffff || z > best) { best = z; bi = cls; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ob > best || (ob == best && oi < bi))) { best = ob; bi = oi; }
      }
      if (lane == 0) {
        s_best[warp] = best;
        s_bi[warp] = bi;
      }
      __syncthreads();
      if (tid == 0) {
        float bb = s_best[0];
        int k = s_bi[0];
        for (int w = 1; w < kThreads / 32; ++w)
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
  return sizeof(float) * ((size_t)6 * P + 2 * J + (size_t)(C > kThreads ? C : kThreads));
}

cudaError_t launch_rnnt_greedy(const float* eproj, const int* lens, const int* off, int batch, int t_max,
                               const float* gtab, const __half* whhT, const __half* wpT, const float* bp,
                               const __half* woT, const float* bo, int C, int P, int J, int max_symbols, int act,
                               int max_tokens, int* tokens, int* frames, int* counts, cudaStream_t s) {
  if (batch <= 0) return cudaSuccess;
  if ((P & 1) || (J & 1) || C < 2 || max_symbols < 1 || max_tokens < 1) return cudaErrorInvalidValue;
  RnntArgs a;
  a.eproj = eproj;
  a.lens = lens;
  a.off = off;
  a.t_max = t_max;
  a.gtab = gtab;
  a.whhT = reinterpret_cast<const __half2*>(whhT);
  a.wpT = reinterpret_cast<const __half2*>(wpT);
  a.bp = bp;
  a.woT = woT;
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
