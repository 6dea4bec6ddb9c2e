// Internal declarations shared by the kernels and the host runtime.
//
// Row layout of the batched activations ("segment layout")
// --------------------------------------------------------
// Clips are packed along one row axis at three time resolutions so that the
// two stride-2 subsampling convs become plain strided GEMMs:
//   encoder rows   clip i occupies [e_i, e_i + L'_i)            (L' valid frames)
//   conv1 rows     clip i occupies [2 e_i + 2, 2 e_i + 2 + L1_i)
//   mel rows       clip i occupies [4 e_i + 6, 4 e_i + 6 + F_i)
// Row r of a stride-2, kernel-5, pad-2 conv reads input rows 2r .. 2r+4,
// i.e. it is centred on input row 2r + 2, which is why the offsets are
// 2 e + 2 and 4 e + 6.  e_{i+1} - e_i is a multiple of 8 and large enough that
// the two rows in front of every clip are outside any clip at both finer
// resolutions (they hold zeros = the convs' zero padding).  Rows outside
// every clip ("gap rows") carry finite junk in the encoder and are never
// read as valid data: attention masks them as keys, the depthwise conv treats
// them as zero padding, the output scatter skips them.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gam {

// Programmatic dependent launch.  The encoder's kernels are launched with the
// programmatic-serialisation attribute, so a kernel's CTAs may be scheduled
// (and do their setup: barriers, TMEM, descriptor prefetch) while the previous
// kernel in the stream is still finishing.  Each such kernel calls pdl_wait()
// before its first global-memory access: it returns once the previous kernel
// has completed and its writes are visible, so the stream order of the data is
// unchanged.  pdl_launch_dependents() lets the next kernel be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Host side: launch with the programmatic-serialisation attribute (unless
// GAM_PDL=0 in the environment), for kernels that call pdl_wait() first.
bool pdl_enabled();
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Device view of the per-call clip table: 5 arrays of B (+1) ints.
struct Clips {
  const int* tab;  // [5][B+1]: e (B+1 entries), F, L1, L2, N
  int B;
  __device__ __forceinline__ int e(int i) const { return __ldg(tab + i); }
  __device__ __forceinline__ int F(int i) const { return __ldg(tab + (B + 1) + i); }
  __device__ __forceinline__ int L1(int i) const { return __ldg(tab + 2 * (B + 1) + i); }
  __device__ __forceinline__ int L2(int i) const { return __ldg(tab + 3 * (B + 1) + i); }
  __device__ __forceinline__ int N(int i) const { return __ldg(tab + 4 * (B + 1) + i); }
  // Largest clip i whose first row at this resolution, scale * e_i + off,
  // is <= r (0 if none): (scale, off) = (1, 0) encoder, (2, 2) conv1,
  // (4, 6) mel rows.  Row r belongs to that clip iff r - (scale e_i + off) is
  // below the clip's length at this resolution.
  __device__ __forceinline__ int find(int r, int scale, int off) const {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (scale * e(mid) + off <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

// Epilogue kinds of the GEMM kernels (C = A . B^T, fp32 accumulation).
enum EpiKind {
  EPI_SWISH = 0,     // out_t[r, n] = swish(acc + b[n])
  EPI_GLU = 1,       // weights interleaved in blocks of 64 (value, gate):
                     //   out_t[r, 64j + c] = (acc_v + b_v) * sigmoid(acc_g + b_g)
  EPI_RESID = 2,     // x[r, n] += alpha * (acc + b[n])        (fp32 residual)
  EPI_QKV = 3,       // scatter to Q/K head-major (padded to 64) and V^T
  EPI_CONV1 = 4,     // out_t = relu(acc + b), zero outside conv1 clip rows
  EPI_CONV2 = 5,     // x (fp32) = relu(acc + b), zero outside encoder clip rows
  EPI_F32 = 6        // out_f32[r, n] = acc + b[n] (n < n_valid, or N when n_valid == 0)
};

struct EpiParams {
  void* out;          // output (type depends on kind)
  float* x;           // fp32 residual stream (EPI_RESID / EPI_CONV2)
  const float* bias;  // [N] fp32
  float alpha;
  int ldo;            // row stride of `out` / `x` in elements
  Clips clips;
  // EPI_QKV
  void* qk;           // [2][H][rows_pad][64]
  void* vt;           // [H][64][rows_pad]
  int rows_pad, n_heads, d_head, d_model;
  int n_valid;        // EPI_F32: columns stored (the padded weight rows beyond it are skipped)
};

// Kernel families for profiling (order = gam_profile_kind_name order).
enum ProfKind {
  PK_FRONTEND = 0, PK_GEMM_SUB = 1, PK_GEMM_FFN_UP = 2, PK_GEMM_FFN_DOWN = 3, PK_GEMM_QKV = 4,
  PK_GEMM_OUT = 5, PK_GEMM_PW1 = 6, PK_GEMM_PW2 = 7, PK_ATTENTION = 8, PK_LAYERNORM = 9,
  PK_DWCONV = 10, PK_CTC_GEMM = 11, PK_CTC_SOFTMAX = 12, PK_CTC_COLLAPSE = 13, PK_MISC = 14,
  PK_RNNT_ENC_PROJ = 15, PK_RNNT_DECODE = 16,
  PK_COUNT = 17
};

// Weight operand of a GEMM: [N, K] row-major (PyTorch Linear layout).
struct WeightOp {
  const void* w;         // float / __half / int8 [N, K]
  const __half* scale;   // int8 only: [N, K/64]
  int dtype;             // 0 f32, 1 f16, 2 int8-g64
  const __half* scale_t; // int8 only: the same scales transposed to [K/64, N]
};

// --- launchers (return cudaGetLastError()) ---------------------------------

// SIMT GEMM: A [M, K] (row stride lda, element type a_dtype 0 f32 / 1 f16),
// optional A2 used for output columns n >= n_split (QKV: rotated input for
// Q/K, plain input for V).
cudaError_t launch_gemm_simt(int a_dtype, const void* A, const void* A2, int n_split, int lda,
                             WeightOp B, int M, int N, int K, int epi, int out_half,
                             const EpiParams& ep, cudaStream_t s);

cudaError_t launch_frontend(const float* audio, int64_t audio_stride, Clips clips, int rows, int packed,
                            int f_max, const float* basis, const float* fb, void* out, int out_half,
                            cudaStream_t s);

// Tensor-core frontend of the fp16 / INT8 modes (frontend_tc.cu), step 1: the
// clips' samples as packed rows of 160 (row 4 e_i + 6 + g = samples 160 g ..
// of clip i, g <= F_i), split into tf32 hi and lo parts; zero rows elsewhere.
cudaError_t launch_audio_split(const float* audio, int64_t audio_stride, Clips clips, int rows, float* hi, float* lo,
                               cudaStream_t s);

cudaError_t launch_layernorm(const float* x, const float* g, const float* b, float eps, void* u, int u_half,
                             int rows, int d, cudaStream_t s);
cudaError_t launch_layernorm_rope(const float* x, const float* g, const float* b, float eps,
                                  const float* cos_tab, const float* sin_tab, Clips clips, void* u,
                                  void* urot, int u_half, int rows, int d, int d_head, cudaStream_t s);
cudaError_t launch_layernorm_chain(float* x, const float* g1, const float* b1, const float* g2,
                                   const float* b2, float eps, void* u, int u_half, int rows, int d,
                                   cudaStream_t s);
// Depthwise conv + folded BN + Swish.  fp16 activations with K 31 / 15 / 5 run the
// persistent TMA-fed form (needs status, the device word a bounded wait that gave
// up sets, and sm_count for its grid); other sizes and fp32 run the tiled forms.
cudaError_t launch_dwconv(const void* g, const float* w, const float* bias, Clips clips, void* out, int t_half,
                          int rows, int d, int K, int sm_count, int* status, cudaStream_t s);
cudaError_t launch_scatter_out(const float* x, Clips clips, float* out, int t_max, int d, cudaStream_t s);
cudaError_t launch_attention_simt(const void* qk, const void* vt, Clips clips, void* o, int t_half,
                                  int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s);
// logits row of frame (b, t): b * t_max + t, or off[b] + t when off (per-clip
// offsets of the compacted valid frames, B + 1 entries) is given.
cudaError_t launch_logsoftmax_argmax(const float* logits, int ld, const int* lens, int batch, int t_max,
                                     int C, float* logp, int* argmax, cudaStream_t s, const int* off = nullptr);
// Valid frames of enc [B, t_max, d] (fp32) compacted to rows off[b] + t and
// split into fp16 hi and lo parts: a[v, c] = hi, a[v, d + c] = lo (x ~= hi + lo).
cudaError_t launch_split_hi_lo(const float* enc, const int* off, int batch, int t_max, int d, int rows,
                               __half* a, cudaStream_t s);
// frames (optional): the first frame of each token's run, -1 after the last token.
cudaError_t launch_collapse(const int* argmax, const int* lens, int batch, int t_max, int blank,
                            int* tokens, int* counts, cudaStream_t s, int* frames = nullptr);
cudaError_t launch_f32_to_f16(const float* in, __half* out, int64_t n, cudaStream_t s);

// Greedy RNNT decoding (rnnt.cu).  eproj [rows][J]: the joint's encoder
// projection per valid frame (row off[b] + t, or b * t_max + t when off is NULL);
// gtab [(C + 1)][4P]: LSTM input gates per symbol (row C: zero start input);
// whh [4P][P], wp [J][P], wo [C][J] fp16, row-major (PyTorch layout), 16-byte
// aligned, P and J multiples of 8 up to 1024; act 0 ReLU, 1 tanh.  order [B]: the
// clips by decreasing length; with it, a head whose slices fit in the shared
// memory of an 8-CTA cluster is decoded by one cluster per clip with resident
// weights, otherwise (or with order NULL, or GAM_RNNT=ring in the environment)
// by one CTA per clip that streams the weights.  status: the device word a
// bounded wait that gave up sets.  Writes tokens / frames ([B][max_tokens], -1
// after the last symbol; frames may be NULL) and counts [B].
size_t rnnt_smem_bytes(int C, int P, int J);
cudaError_t launch_rnnt_greedy(const float* eproj, const int* lens, const int* off, const int* order, int batch,
                               int t_max, const float* gtab, const __half* whh, const __half* wp, const float* bp,
                               const __half* wo, const float* bo, int C, int P, int J, int max_symbols, int act,
                               int max_tokens, int* tokens, int* frames, int* counts, int* status, cudaStream_t s);

}  // namespace gam

#include <string>

namespace gam {

// Error text of calls that take no context, returned by gam_last_error(NULL).
void set_context_free_error(const std::string& msg);

}  // namespace gam
