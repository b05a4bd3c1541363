// fvattn_route_static_scratch: fvattn_route for callers that cannot allocate device memory.
//
// Some hosts hand a kernel library nothing but the pointers of its inputs and outputs: a
// serving runtime that owns every byte of device memory through its own fixed-budget pool,
// or a plugin interface of an inference engine whose contract forbids calls into the CUDA
// allocator. Such callers cannot provide the workspace that fvattn_route needs. This entry
// point runs the same router kernels with their scratch in a file-scope device array of
// FVATTN_STATIC_SCRATCH_BYTES, which every GPU that loads the library keeps until exit.
//
// Device addresses: in host code the name of a __device__ array is only a host-side
// stand-in; a kernel given that name would fault, or on a GPU that can reach host memory
// silently use the wrong memory. So, once per device and with that device current, the
// first call looks up the real address with cudaGetSymbolAddress and caches it.
#include <mutex>

#include "common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_route_scratch[FVATTN_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FVATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return FVATTN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FVATTN_OK;
}

}  // namespace

extern "C" int fvattn_route_static_scratch(const void* Q, const void* K, const fvattn_shape* shape,
                                           const fvattn_route_cfg* cfg, const fvattn_csr* out,
                                           fvattn_stream_t stream) {
  const size_t need = fvattn_route_workspace_bytes(shape, cfg);
  if (need == 0) return FVATTN_ERR_INVALID;
  if (need > (size_t)FVATTN_STATIC_SCRATCH_BYTES) return FVATTN_ERR_CAPACITY;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != FVATTN_OK) return st;
  // Nothing in the scratch has to start at zero: every word the router reads there is
  // written earlier in the same call (block means, selection bitmasks, row counts).
  return fvattn_route(Q, K, shape, cfg, out, scratch, (size_t)FVATTN_STATIC_SCRATCH_BYTES, stream);
}
