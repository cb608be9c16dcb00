// qi21_attn_cached_noalloc: the target-only cached step for callers that may
// not allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they run attention: plugin hosts that hand a library only a stream and
// the tensors, serving loops that reserve all memory at start-up and forbid
// later allocation, and latency-critical loops where an allocation would
// synchronise the device.  This entry point gives them the cached step with
// its scratch memory built into the library: a file-scope device array of
// kNoAllocScratchBytes (32 MiB), which every GPU that loads the library holds
// until the process exits.  The caller passes inputs and outputs only.
#include <mutex>

#include "../../include/qi21.h"
#include "qi21_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kNoAllocMaxDevices = 64;

// The scratch itself.  Host code must not use this name as a device address:
// on the host it is only a stand-in; the device address comes from
// cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

}  // namespace

extern "C" qi21_status qi21_attn_cached_noalloc(int32_t B, int32_t H, int64_t P, int64_t T,
                                                qi21_dtype dt, const void* q, const void* k,
                                                const void* v, const int32_t* pos_tgt,
                                                const void* k_cache, const void* v_cache, void* o,
                                                void* stream) {
  const size_t need = qi21_attn_cached_workspace_size(B, H, P, T, dt);
  if (need > kNoAllocScratchBytes)
    return qi21::report_error(
        QI21_ERR_INVALID_ARG,
        "qi21_attn_cached_noalloc: B*H*T too large for the built-in scratch (%zu bytes needed, "
        "%zu available); call qi21_attn_cached with a workspace instead",
        need, kNoAllocScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return qi21::report_error(QI21_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return qi21::report_error(QI21_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      // First call on this device (the current one): resolve the array's
      // device address.
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess)
        return qi21::report_error(QI21_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  // The scratch keeps the previous call's contents; the status header must
  // start at zero.
  e = cudaMemsetAsync(scratch, 0, QI21_WORKSPACE_HEADER_BYTES, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return qi21::report_error(QI21_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  return qi21_attn_cached(B, H, P, T, dt, q, k, v, pos_tgt, k_cache, v_cache, o, scratch,
                          kNoAllocScratchBytes, stream);
}
