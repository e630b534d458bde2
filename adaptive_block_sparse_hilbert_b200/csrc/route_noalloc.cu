// fva_route_noalloc: routing for callers that cannot allocate device memory.
//
// Some callers have no way to hand libfva a workspace: a plugin loaded into a host
// application whose allocator owns all device memory and exposes none of it, a service
// that forbids any allocation after start-up so its memory footprint stays fixed, or a
// caller whose only buffers are the inputs and outputs it was given. This entry point
// runs the same routing kernels as fva_route, but their scratch (block logits, kept
// bitmasks, row counts, per-head loads, and the pooled Q/K when they are not passed
// in) lives in one fixed device array that belongs to the library.
//
// The array is a file-scope __device__ variable of FVA_ROUTE_NOALLOC_SCRATCH_BYTES; every
// GPU that loads the library holds it until the process exits. Host code cannot use the
// array's name as a device address (on the host it names a host-side stand-in), so the
// first call on each device looks up the real address with cudaGetSymbolAddress while
// that device is current and caches it.
#include <mutex>

#include "fva_internal.cuh"

namespace fva {

static __device__ __align__(256) uint8_t g_route_scratch[FVA_ROUTE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
}  // namespace

// Device address of the scratch array on the current device (looked up once per device).
static cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace fva

extern "C" int fva_route_noalloc(const fva_shape* s, const void* q_bhnd_dev, const void* k_bhnd_dev,
                                 const double* pooled_q_dev, const double* pooled_k_dev, double p, int k_floor,
                                 int order, const fva_mask* mask, int32_t* dev_status, fva_stream_t stream) {
  if (!s) return FVA_ERR_INVALID_ARG;
  if ((pooled_q_dev == nullptr) != (pooled_k_dev == nullptr)) return FVA_ERR_INVALID_ARG;
  const int need_pool = (pooled_q_dev && pooled_k_dev) ? 0 : 1;
  const size_t need = fva_route_workspace_bytes(s, need_pool);
  if (need == 0) return FVA_ERR_UNSUPPORTED_SHAPE;
  if (need > FVA_ROUTE_NOALLOC_SCRATCH_BYTES) return FVA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  if (fva::scratch_address(&scratch) != cudaSuccess) return FVA_ERR_CUDA;
  return fva_route(s, q_bhnd_dev, k_bhnd_dev, pooled_q_dev, pooled_k_dev, p, k_floor, order, mask, scratch,
                   FVA_ROUTE_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
