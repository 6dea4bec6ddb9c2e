// Tensor-core kernels (placeholder dispatch: CUDA-core path until the tcgen05 kernels are enabled).
#include "gemm_tc.cuh"

namespace gam {

bool tc_supported(int, int, int, int, int) { return false; }

cudaError_t launch_gemm_tc(TcGemmCache*, const void*, const void*, int, int, WeightOp, int, int, int, int,
                           const EpiParams&, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_attention(TcGemmCache*, const void* qk, const void* vt, Clips clips, void* o, int t_half,
                             int rows_pad, int n_heads, int d_head, int t_max, cudaStream_t s) {
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
