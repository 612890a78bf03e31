// avey_rank_static.cu -- avey_rank for callers that cannot allocate device
// memory.
//
// Some callers have no way to hand this library a workspace: a plugin ABI that
// passes only the input and output buffers, or a host that owns every
// allocation and forbids cudaMalloc on the calling path (an allocation there
// would also synchronise the device).  avey_rank_static serves them: it runs
// exactly the kernels of avey_rank, but its scratch (the per-token inverse
// norms and the split-score matrix) lives in the file-scope device array
// below instead of a caller-provided workspace.
//
// The array is a fixed 16 MiB that every GPU which loads this library keeps
// until the process exits.  The host-side name of the array is only a
// stand-in, never a device address, so every call looks up the array's address
// on the current device (cudaGetSymbolAddress, which allocates nothing); the
// first call on a device may load the library's device code there, so that
// first call should come before any stream capture.  All calls share the
// array and it keeps the previous call's contents; nothing in it needs to
// start at zero because every call writes each scratch entry it reads.  Calls
// whose kernels overlap on the GPU (different streams, no ordering between
// them) race on the array.
#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_rank_scratch[kScratchBytes];

// Device address of the scratch array on the current device, looked up on
// every call (a primary-context reset may move the module, so no address is
// cached); nullptr with the detail set on failure.
unsigned char *scratch_for_current_device() {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_rank_scratch);
  if (e != cudaSuccess || p == nullptr) {
    set_detail("avey_rank_static: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    return nullptr;
  }
  return static_cast<unsigned char *>(p);
}

}  // namespace
}  // namespace avey

extern "C" size_t avey_rank_static_max_scratch_bytes(void) { return avey::kScratchBytes; }

extern "C" avey_status avey_rank_static(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                        int k, int32_t *idx, float *w, avey_stream_t stream) {
  using namespace avey;
  // Host-side checks first (the same as avey_rank's, so that an invalid shape
  // is reported as such), then the size check, all before any CUDA call.
  AVEY_REQUIRE(x && idx && w, AVEY_ERR_INVALID_ARG, "avey_rank_static: null pointer");
  {
    const avey_status sh = check_rank_shape("avey_rank_static", dt, B, N, d, S, k);
    if (sh != AVEY_OK) return sh;
  }
  const size_t need = avey_rank_workspace_bytes(dt, B, N, d, S);
  AVEY_REQUIRE(need <= kScratchBytes, AVEY_ERR_UNSUPPORTED,
               "avey_rank_static: this shape needs %zu bytes of scratch, more than the fixed "
               "%zu-byte device array; call avey_rank with a workspace instead",
               need, kScratchBytes);
  unsigned char *scratch = scratch_for_current_device();
  if (!scratch) return AVEY_ERR_CUDA;
  // Same kernels, same launch configuration as avey_rank; the scratch array
  // takes the place of the workspace (the split scores go to its second part).
  return avey_rank(x, dt, B, N, d, S, k, idx, w, nullptr, scratch, kScratchBytes, stream);
}
