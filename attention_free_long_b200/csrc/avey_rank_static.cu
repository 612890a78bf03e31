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
// until the process exits.  Its device address is looked up once per device,
// on the first call made with that device current (cudaGetSymbolAddress; the
// host-side name of the array is only a stand-in, never a device address), so
// that first call should come before any stream capture.  All calls share the
// array and it keeps the previous call's contents; nothing in it needs to
// start at zero because every call writes each scratch entry it reads.  Calls
// whose kernels overlap on the GPU (different streams, no ordering between
// them) race on the array.
#include <mutex>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_rank_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per
// device); nullptr with the detail set on failure.
unsigned char *scratch_for_current_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_detail("avey_rank_static: cudaGetDevice failed: %s", cudaGetErrorString(e));
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rank_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_detail("avey_rank_static: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      return nullptr;
    }
    g_scratch_ptr[dev] = static_cast<unsigned char *>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace avey

extern "C" size_t avey_rank_static_max_scratch_bytes(void) { return avey::kScratchBytes; }

extern "C" avey_status avey_rank_static(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                        int k, int32_t *idx, float *w, avey_stream_t stream) {
  using namespace avey;
  // Host-side checks first; the size check runs before any CUDA call.
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16, AVEY_ERR_UNSUPPORTED,
               "avey_rank_static: dtype %d unsupported (F32 or BF16)", int(dt));
  AVEY_REQUIRE(B >= 1 && N >= 1 && d >= 1 && S >= 1, AVEY_ERR_INVALID_ARG,
               "avey_rank_static: sizes must be >= 1");
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
