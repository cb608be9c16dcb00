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
#include "../../include/qi21.h"
#include "qi21_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

// The scratch itself.  Host code must not use this name as a device address:
// on the host it is only a stand-in; the device address comes from
// cudaGetSymbolAddress below.  Static storage: it is zero when the module is
// loaded on a device, so its status header starts at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

namespace qi21 {

// Device address of the built-in scratch on the current device.  Resolved on
// every call (cheap once the module is loaded), so a context that was reset
// and re-created gets the array's new address.  The first call on a device
// loads the module there: it must not happen during a stream capture.
cudaError_t noalloc_scratch(void** ptr) {
  *ptr = nullptr;
  return cudaGetSymbolAddress(ptr, g_noalloc_scratch);
}

}  // namespace qi21

extern "C" qi21_status qi21_attn_cached_noalloc(int32_t B, int32_t H, int64_t P, int64_t T,
                                                qi21_dtype dt, const void* q, const void* k,
                                                const void* v, const int32_t* pos_tgt,
                                                const void* k_cache, const void* v_cache, void* o,
                                                void* stream) {
  const size_t need = qi21::attn_cached_workspace_min(B, H, T, dt);
  if (need > kNoAllocScratchBytes)
    return qi21::report_error(
        QI21_ERR_INVALID_ARG,
        "qi21_attn_cached_noalloc: B*H*T too large for the built-in scratch (%zu bytes needed, "
        "%zu available); call qi21_attn_cached with a workspace instead",
        need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  const cudaError_t e = qi21::noalloc_scratch(&scratch);
  if (e != cudaSuccess)
    return qi21::report_error(QI21_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
  // Nothing is cleared here: the status word is only ever set by a device
  // wait that ran out and is cleared by qi21_workspace_status(NULL, ...); the
  // schedule counter is reset by the call's own first kernel.  So a call that
  // fails its argument checks enqueues nothing, and a recorded timeout stays
  // readable until it is read.
  return qi21_attn_cached(B, H, P, T, dt, q, k, v, pos_tgt, k_cache, v_cache, o, scratch,
                          kNoAllocScratchBytes, stream);
}
