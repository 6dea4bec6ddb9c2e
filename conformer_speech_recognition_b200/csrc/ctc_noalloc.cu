// Greedy CTC decoding that allocates nothing: gam_ctc_collapse_noalloc.
//
// Some callers cannot call cudaMalloc at all: code that runs where the device
// allocator must not be entered (its calls can synchronise the device, which a
// latency-bound audio path cannot afford), plug-ins hosted by a framework that
// owns every byte of device memory, or callers that have no CUDA context of
// their own to create a gam_ctx with.  This entry point needs no context and
// no allocation: the caller passes the inputs and outputs, and the per-frame
// argmax that the collapse reads lives in a fixed array in this file.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds GAM_NOALLOC_MAX_FRAMES * 4 bytes (4 MiB) of it until the
// process exits.  Host code cannot use the array's name as a device address;
// on the first call on a device (with that device current) the address is
// looked up once with cudaGetSymbolAddress and cached together with the
// device's current CUDA context: after a cudaDeviceReset the device gets a new
// context (and the module a new load), so the lookup is done again there
// instead of reusing an address that no longer exists.  Every call on a device
// shares the one array: calls whose GPU work overlaps (two streams, or two
// threads) race on it.  The argmax kernel writes every entry the collapse
// kernel later reads, so nothing has to be cleared between calls.
#include <cuda.h>

#include <mutex>
#include <string>

#include "../../include/gam.h"
#include "common.cuh"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) int g_noalloc_argmax[GAM_NOALLOC_MAX_FRAMES];

std::mutex g_mu;
int* g_addr[kMaxDevices] = {};
CUcontext g_addr_ctx[kMaxDevices] = {};  // the context each cached address belongs to

// The calling thread's current CUDA context (driver entry point resolved through
// the runtime, so the library links against cudart only).
cudaError_t current_context(CUcontext* out) {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (Fn) nullptr;
    return reinterpret_cast<Fn>(f);
  }();
  if (!fn) return cudaErrorNotSupported;
  return fn(out) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

gam_status fail(gam_status s, const std::string& msg) {
  gam::set_context_free_error(msg);
  return s;
}

}  // namespace

extern "C" gam_status gam_ctc_collapse_noalloc(const float* logits_dev, const int32_t* lengths_dev, int batch,
                                               int t_max, int n_classes, int32_t* tokens_dev, int32_t* counts_dev,
                                               void* stream) {
  gam::set_context_free_error("");
  if (!logits_dev || !lengths_dev || !tokens_dev || !counts_dev)
    return fail(GAM_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || t_max < 1 || n_classes < 2) return fail(GAM_ERR_INVALID_ARG, "batch, t_max >= 1 and n_classes >= 2");
  if ((int64_t)batch * t_max > GAM_NOALLOC_MAX_FRAMES)
    return fail(GAM_ERR_CAPACITY, "batch * t_max = " + std::to_string((int64_t)batch * t_max) +
                                      " frames exceeds the fixed scratch of " +
                                      std::to_string(GAM_NOALLOC_MAX_FRAMES) + " frames");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GAM_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(GAM_ERR_UNSUPPORTED_DEVICE, "device index above 63");
  int* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    CUcontext ctx = nullptr;
    if (g_addr[dev]) {
      e = current_context(&ctx);
      if (e != cudaSuccess) return fail(GAM_ERR_CUDA, std::string("cuCtxGetCurrent: ") + cudaGetErrorString(e));
    }
    if (!g_addr[dev] || ctx != g_addr_ctx[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_argmax);  // also makes the device's primary context current
      if (e != cudaSuccess)
        return fail(GAM_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      e = current_context(&ctx);
      if (e != cudaSuccess) return fail(GAM_ERR_CUDA, std::string("cuCtxGetCurrent: ") + cudaGetErrorString(e));
      g_addr[dev] = static_cast<int*>(p);
      g_addr_ctx[dev] = ctx;
    }
    scratch = g_addr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = gam::launch_logsoftmax_argmax(logits_dev, n_classes, lengths_dev, batch, t_max, n_classes, nullptr, scratch, s);
  if (e == cudaSuccess) e = gam::launch_collapse(scratch, lengths_dev, batch, t_max, n_classes - 1, tokens_dev, counts_dev, s);
  if (e != cudaSuccess) return fail(GAM_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return GAM_OK;
}
