// waits_score_static: waits_score for callers that cannot allocate device
// memory.  Some hosts of this library never call cudaMalloc themselves: a
// plugin inside an inference engine whose memory pool owns every byte of the
// device, code that runs inside a region where allocation is forbidden or
// would synchronise the device, or a C caller without an allocator of its
// own.  They can still hand over Q, K and the scores buffer, but not the
// scorer's scratch (work plan, row biases, partial sums).  This entry point
// keeps that scratch in one file-scope device array instead, sized for one
// Llama-3.1-8B-shaped layer of 32768 tokens.
#include <mutex>

#include "waits_internal.cuh"

namespace {

// Scratch shared by every call on a device; the planner kernel rewrites all
// of it (plan, counters, status word) at the start of each call, so nothing
// has to be cleared between calls.  Every device that loads the library holds
// its own copy until the process exits.
__device__ __align__(256) unsigned char g_static_scratch[WAITS_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  In host code
// the array's name denotes a host-side shadow, not device memory, so the
// address is looked up once per device with that device current.
waits_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WAITS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return WAITS_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return WAITS_OK;
}

}  // namespace

extern "C" waits_status waits_score_static(const waits_shape* shape, const void* Q,
                                           const void* K, float a, int32_t b, float* scores,
                                           void* stream) {
  size_t need = 0;
  waits_status st = waits_workspace_size(shape, &need);
  if (st != WAITS_OK) return st;
  if (need > (size_t)WAITS_STATIC_WORKSPACE_BYTES) return WAITS_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != WAITS_OK) return st;
  return waits_score(shape, Q, K, a, b, scores, scratch, (size_t)WAITS_STATIC_WORKSPACE_BYTES,
                     stream);
}
