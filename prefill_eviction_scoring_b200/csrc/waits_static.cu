// waits_score_static: waits_score for callers that cannot allocate device
// memory.  Some hosts of this library never call cudaMalloc themselves: a
// plugin inside an inference engine whose memory pool owns every byte of the
// device, code that runs inside a region where allocation is forbidden or
// would synchronise the device, or a C caller without an allocator of its
// own.  They can still hand over Q, K and the scores buffer, but not the
// scorer's scratch (work plan, row partials, counters, status word).  This
// entry point keeps that scratch in one file-scope device array instead,
// sized for one Llama-3.1-8B-shaped layer of 32768 tokens.
#include <cuda.h>

#include <mutex>

#include "waits_internal.cuh"

namespace {

// Scratch shared by every call on a device.  Nothing has to be cleared
// between calls: every piece of it a call reads was written earlier in the
// same call -- the status word by the first pass-1 CTA (or by the planner
// kernel, which also rewrites the plan and the pass-2 counters when it
// runs), the row partials by the pass-1 units that own them.  Every device
// that loads the library holds its own copy until the process exits.
__device__ __align__(256) unsigned char g_static_scratch[WAITS_STATIC_WORKSPACE_BYTES];

// The array's device address, cached per device and per CUDA context: a
// device reset (or any teardown of the primary context) loads the module
// again at another address, so a cached pointer is reused only while the
// context it was looked up in is still the current one (contexts are told
// apart by their unique 64-bit id, which the driver never reuses).
typedef CUresult (*CtxGetCurrentFn)(CUcontext* ctx);
typedef CUresult (*CtxGetIdFn)(CUcontext ctx, unsigned long long* id);

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
struct Cached {
  void* ptr;
  unsigned long long ctx_id;
};
Cached g_cache[kMaxDevices] = {};

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Id of the context current on this thread (0 if none or unknown).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_static_scratch on the current device.  In host code
// the array's name denotes a host-side stand-in, not device memory, so the
// address is looked up with cudaGetSymbolAddress, with the device current,
// once per device and context.
waits_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WAITS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  const unsigned long long id = current_ctx_id();
  Cached& c = g_cache[dev];
  if (!c.ptr || id == 0 || c.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return WAITS_ERR_CUDA;
    // the lookup makes the runtime's context current if none was
    c.ptr = p;
    c.ctx_id = id != 0 ? id : current_ctx_id();
  }
  *out = c.ptr;
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

extern "C" waits_status waits_read_static_status(void* stream, uint32_t* status_bits) {
  if (!status_bits) return WAITS_ERR_ARG;
  void* scratch = nullptr;
  const waits_status st = scratch_address(&scratch);
  if (st != WAITS_OK) return st;
  return waits_read_device_status(scratch, (size_t)WAITS_STATIC_WORKSPACE_BYTES, stream,
                                  status_bits);
}
