// Tensor-core (tcgen05 / TMEM / TMA) kernels: GEMM with fused epilogues and
// masked flash attention.  Host-side interface used by the runtime.
#pragma once

#include "common.cuh"

namespace gam {

// Per-context state of the tensor-core kernels (tensor-map cache, status word).
struct TcGemmCache {
  int* status = nullptr;  // device word set when a bounded wait gives up
  int sm_count = 148;
  // fp16 GEMM tiles: 0 single-CTA only, 1 single- or paired-CTA (cta_group::2)
  // tiles, whichever is cheaper, 2 paired-CTA tiles wherever one applies
  int pair_mode = 1;
  // Test hook, consumed by the next tensor-core GEMM launch: its bounded waits
  // give up after debug_limit_ns, and (single-CTA tiles) its producer never
  // issues the loads of the debug_skip-th k-block it handles, so the wait for
  // that stage runs out.  -1 / 0: off.
  int debug_skip = -1;
  uint64_t debug_limit_ns = 0;
  // quantised-weight GEMMs: 128-row A tiles per CTA tile (2: one converted B stage
  // feeds two accumulators; 1: one), GAM_QB_TILES=m1|m2
  int qb_mt = 2;
  // fp16 GEMMs of at most 256 rows: split K over a cluster of 2 .. 4 CTAs when that
  // puts more SMs on the weight stream (GAM_SPLITK=0 turns it off)
  bool splitk = true;
};

// Resolves the driver's tensor-map encoder and allocates the status word.
cudaError_t tc_init(TcGemmCache* cache, int device);

// True when the tensor-core GEMM handles this operand / shape / epilogue combination.
bool tc_supported(int a_dtype, int b_dtype, int N, int K, int epi);

struct TileShape {
  bool pair;   // paired-CTA (cta_group::2) tile of 256 rows, else 128 rows on one SM
  int width;   // output columns per tile (256, 192 or 128); 0: no shape applies
  int mt = 1;  // single-CTA tiles: 128-row A tiles per tile (2: quantised weights, 256 x 128)
};

// The tile shape launch_gemm_tc uses.  variant: -1 any, 0 single-CTA only,
// 1 paired-CTA only (fp16 weights); width: 0 any, else 256, 192 or 128;
// n_split > 0: output columns from n_split on read a second A operand, so a
// tile's width must divide n_split.
TileShape choose_tile(const TcGemmCache* cache, int M, int N, int epi, bool int8_weights, int variant, int width,
                      int n_split = 0);

// One tensor-core GEMM with a fused epilogue.  variant as for choose_tile, plus
// 2: split K over a cluster (fp16 weights, at most 256 rows; fails where no split
// applies).  With variant -1, width 0 and at most 256 rows the library splits K
// by itself when that helps (TcGemmCache::splitk).
cudaError_t launch_gemm_tc(TcGemmCache* cache, const void* A, const void* A2, int n_split, int lda, WeightOp B,
                           int M, int N, int K, int epi, const EpiParams& ep, cudaStream_t s, int variant = -1,
                           int width = 0);

// Masked multi-head attention on tensor cores (fp16 Q/K/V^T, see attention_tc.cu).
cudaError_t launch_attention_tc(TcGemmCache* cache, const void* qk, const void* vt, Clips clips, void* o,
                                int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s);

// The same with 64-key blocks, the score tile double-buffered in TMEM and P kept
// in TMEM for the P.V product (attention_tc2.cu).
cudaError_t launch_attention_tc2(TcGemmCache* cache, const void* qk, const void* vt, Clips clips, void* o,
                                 int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s);

// Masked multi-head attention: tensor cores for fp16 activations (the double-buffered
// form unless GAM_ATTN=1 in the environment), CUDA cores for fp32.
cudaError_t launch_attention(TcGemmCache* cache, const void* qk, const void* vt, Clips clips, void* o, int t_half,
                             int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s);

// Tensor-core frontend (frontend_tc.cu), step 2: 3xTF32 windowed DFT of the
// frames (pairs of split rows, split_rows >= rows + 1) against the basis
// [384][320] (hi and lo parts), power, filterbank fb [161][64] over the nonzero
// rows fb_range (int pairs per mel bin) and log(clip(., 1e-9, 1e9)).  mode 0:
// out = fp16 packed mel rows [rows][64], zero outside clips; mode 1: out = fp32
// [B][f_max][64], written for valid frames only.
cudaError_t launch_dft_mel(TcGemmCache* cache, const float* hi, const float* lo, int split_rows,
                           const float* basis_hi, const float* basis_lo, const float* fb, const int* fb_range,
                           Clips clips, int rows, int mode, int f_max, void* out, cudaStream_t s);

cudaError_t tc_read_status(TcGemmCache* cache, int* status);
cudaError_t tc_reset_status(TcGemmCache* cache);
void tc_release(TcGemmCache* cache);

}  // namespace gam
