// avey_abi.cu -- host-side utilities of libavey.so: status reporting, error
// details, launch counting and the kernel trace, SM count, and TMA tensor-map
// encoding.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "avey_common.cuh"

namespace avey {

// Device status word: kernels record the first failure here (no trap, no
// assert); avey_device_status() reads and clears it.
static __device__ int g_status_word;

namespace {
thread_local char t_detail[512] = {0};
std::atomic<uint64_t> g_launches{0};
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}
}  // namespace

void set_detail(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_detail, sizeof(t_detail), fmt, ap);
  va_end(ap);
}

int *device_status_word() {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) == cudaSuccess) g_status_ptr[dev] = static_cast<int *>(p);
  }
  return g_status_ptr[dev];
}

// Kernel trace: while active, every launch records the next of the library's
// own events on the launch's stream and keeps the kernel's name.  The events
// are created by this library's CUDA runtime (handles made by another runtime
// instance, such as the caller's, are not valid here) and reused.
namespace {
constexpr int kTraceName = 48;
constexpr int kTraceMax = 4096;
struct Trace {
  std::mutex mu;
  std::atomic<bool> on{false};
  cudaEvent_t events[kTraceMax + 1] = {};  // [0] the start, [i + 1] after launch i
  int created = 0;                         // events created so far
  int device = -1;                         // device the events belong to
  int capacity = 0;
  int count = 0;       // launches seen since avey_trace_begin
  int record_err = 0;  // first cudaEventRecord failure
  char names[kTraceMax][kTraceName];
};
Trace g_trace;
}  // namespace

void count_launch(const char *name, cudaStream_t stream) {
  g_launches.fetch_add(1);
  if (!g_trace.on.load(std::memory_order_acquire)) return;
  std::lock_guard<std::mutex> lk(g_trace.mu);
  if (!g_trace.on.load(std::memory_order_relaxed)) return;
  const int i = g_trace.count++;
  if (i < g_trace.capacity) {
    snprintf(g_trace.names[i], kTraceName, "%s", name ? name : "?");
    const cudaError_t e = cudaEventRecord(g_trace.events[i + 1], stream);
    if (e != cudaSuccess && !g_trace.record_err) g_trace.record_err = static_cast<int>(e);
  }
}

int sm_count() {
  const int dev = current_device();
  if (dev < 0) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = v > 0 ? v : 148;
  }
  return g_sms[dev];
}

bool encode_map(CUtensorMap *map, bool fp32, const void *base, uint64_t inner, uint64_t rows,
                uint64_t batch, uint64_t row_stride_bytes, uint64_t batch_stride_bytes,
                uint32_t box_inner, uint32_t box_rows, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_detail("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  const cuuint64_t dims[3] = {inner, rows, batch};
  const cuuint64_t strides[2] = {row_stride_bytes, batch_stride_bytes};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_detail("cuTensorMapEncodeTiled failed (%d): inner=%llu rows=%llu batch=%llu box=%ux%u", int(r),
               (unsigned long long)inner, (unsigned long long)rows, (unsigned long long)batch,
               box_inner, box_rows);
    return false;
  }
  return true;
}

bool encode_bf16_map(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                     uint64_t batch, uint64_t row_stride_bytes, uint64_t batch_stride_bytes,
                     uint32_t box_rows) {
  return encode_map(map, false, base, inner, rows, batch, row_stride_bytes, batch_stride_bytes, 64,
                    box_rows, 128);
}

// Self-test of the bounded waits: one warp waits on an mbarrier that nothing
// ever arrives on, through the same wait routine the tcgen05 kernels use,
// with a short limit; on expiry it records the timeout and returns.
__global__ void wait_timeout_probe(uint64_t limit_ns, int *status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (!mbar_wait_limit(smem_u32(&bar), 0, &abort_flag, limit_ns))
      record_status(status, AVEY_ERR_DEVICE_TIMEOUT);
    // complete the barrier's phase so nothing is left pending
    mbar_arrive(smem_u32(&bar));
  }
}

}  // namespace avey

extern "C" {

avey_status avey_selftest_wait_timeout(uint32_t limit_us, avey_stream_t stream) {
  AVEY_REQUIRE(limit_us >= 1 && limit_us <= 2000000, AVEY_ERR_INVALID_ARG,
               "avey_selftest_wait_timeout: limit_us must be in [1, 2000000]");
  int *st = avey::device_status_word();
  AVEY_REQUIRE(st != nullptr, AVEY_ERR_CUDA, "avey_selftest_wait_timeout: no device status word");
  avey::wait_timeout_probe<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull, st);
  AVEY_CHECK_LAUNCH("wait_timeout_probe", reinterpret_cast<cudaStream_t>(stream));
  return AVEY_OK;
}


avey_status avey_device_status(avey_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    avey::set_detail("cudaStreamSynchronize: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, avey::g_status_word, sizeof(int));
  if (e != cudaSuccess) {
    avey::set_detail("reading the device status word: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(avey::g_status_word, &zero, sizeof(int));
    if (e != cudaSuccess) {
      avey::set_detail("clearing the device status word: %s", cudaGetErrorString(e));
      return AVEY_ERR_CUDA;
    }
  }
  return static_cast<avey_status>(v);
}

const char *avey_status_string(avey_status s) {
  switch (s) {
    case AVEY_OK: return "AVEY_OK";
    case AVEY_ERR_INVALID_ARG: return "AVEY_ERR_INVALID_ARG";
    case AVEY_ERR_UNSUPPORTED: return "AVEY_ERR_UNSUPPORTED";
    case AVEY_ERR_CUDA: return "AVEY_ERR_CUDA";
    case AVEY_ERR_DEVICE_TIMEOUT: return "AVEY_ERR_DEVICE_TIMEOUT";
    case AVEY_ERR_DEVICE_BOUNDS: return "AVEY_ERR_DEVICE_BOUNDS";
  }
  return "AVEY_ERR_UNKNOWN";
}

const char *avey_last_error_detail(void) { return avey::t_detail; }

uint64_t avey_kernel_launches(void) { return avey::g_launches.load(); }

avey_status avey_trace_begin(int capacity, avey_stream_t stream) {
  using avey::g_trace;
  AVEY_REQUIRE(capacity >= 1 && capacity <= avey::kTraceMax, AVEY_ERR_INVALID_ARG,
               "avey_trace_begin: capacity must be in [1, %d] (got %d)", avey::kTraceMax, capacity);
  std::lock_guard<std::mutex> lk(g_trace.mu);
  AVEY_REQUIRE(!g_trace.on.load(), AVEY_ERR_INVALID_ARG, "avey_trace_begin: a trace is active");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  AVEY_REQUIRE(e == cudaSuccess, AVEY_ERR_CUDA, "avey_trace_begin: cudaGetDevice: %s",
               cudaGetErrorString(e));
  AVEY_REQUIRE(g_trace.device < 0 || g_trace.device == dev, AVEY_ERR_UNSUPPORTED,
               "avey_trace_begin: the trace events belong to device %d, not %d", g_trace.device,
               dev);
  g_trace.device = dev;
  while (g_trace.created < capacity + 1) {
    e = cudaEventCreate(&g_trace.events[g_trace.created]);
    AVEY_REQUIRE(e == cudaSuccess, AVEY_ERR_CUDA, "avey_trace_begin: cudaEventCreate: %s",
                 cudaGetErrorString(e));
    ++g_trace.created;
  }
  e = cudaEventRecord(g_trace.events[0], reinterpret_cast<cudaStream_t>(stream));
  AVEY_REQUIRE(e == cudaSuccess, AVEY_ERR_CUDA, "avey_trace_begin: cudaEventRecord: %s",
               cudaGetErrorString(e));
  g_trace.capacity = capacity;
  g_trace.count = 0;
  g_trace.record_err = 0;
  g_trace.on.store(true, std::memory_order_release);
  return AVEY_OK;
}

int avey_trace_end(void) {
  using avey::g_trace;
  std::lock_guard<std::mutex> lk(g_trace.mu);
  if (!g_trace.on.load()) {
    avey::set_detail("avey_trace_end: no trace is active");
    return -1;
  }
  g_trace.on.store(false, std::memory_order_release);
  if (g_trace.record_err) {
    avey::set_detail("avey_trace_end: cudaEventRecord failed: %s",
                     cudaGetErrorString(static_cast<cudaError_t>(g_trace.record_err)));
    return -1;
  }
  return g_trace.count;
}

const char *avey_trace_kernel_name(int i) {
  using avey::g_trace;
  std::lock_guard<std::mutex> lk(g_trace.mu);
  if (g_trace.on.load() || i < 0 || i >= g_trace.capacity || i >= g_trace.count) return nullptr;
  return g_trace.names[i];
}

avey_status avey_trace_kernel_ms(int i, float *ms) {
  using avey::g_trace;
  AVEY_REQUIRE(ms != nullptr, AVEY_ERR_INVALID_ARG, "avey_trace_kernel_ms: null output");
  std::lock_guard<std::mutex> lk(g_trace.mu);
  AVEY_REQUIRE(!g_trace.on.load(), AVEY_ERR_INVALID_ARG, "avey_trace_kernel_ms: a trace is active");
  AVEY_REQUIRE(i >= 0 && i < g_trace.capacity && i < g_trace.count, AVEY_ERR_INVALID_ARG,
               "avey_trace_kernel_ms: launch %d was not traced", i);
  const cudaError_t e = cudaEventElapsedTime(ms, g_trace.events[i], g_trace.events[i + 1]);
  AVEY_REQUIRE(e == cudaSuccess, AVEY_ERR_CUDA, "avey_trace_kernel_ms: cudaEventElapsedTime: %s",
               cudaGetErrorString(e));
  return AVEY_OK;
}

}  // extern "C"
