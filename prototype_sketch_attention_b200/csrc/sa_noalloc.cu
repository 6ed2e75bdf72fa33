// sa_sketch_forward_noalloc: the Sketch Attention forward for callers that cannot
// allocate device memory.
//
// Some callers have no way to allocate. Examples: code that runs under an allocator
// that forbids new device allocations after start-up (a serving process that reserved
// all of its memory up front, or a framework's arena that must not grow), and hosts
// where the calling thread may not call cudaMalloc at all. For them, the forward's
// scratch memory lives in one file-scope device array, reserved once for the lifetime of
// the process on every GPU that uses this entry point. The caller passes inputs and
// outputs as for sa_sketch_forward and no workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "sa_internal.h"
#include "sa_sketch.h"

namespace {

// Scratch for one forward call, shared by every call on the same device. Its contents
// persist between calls; each call initialises every byte it reads (the first kernel of
// the forward resets the status word, and every partial sum the later kernels read is
// written earlier in the same call), so nothing has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array for the current device: host code only knows a
// host-side stand-in for the symbol, so the address comes from cudaGetSymbolAddress,
// once per device, with that device current.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SA_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SA_OK;
}

}  // namespace

extern "C" int sa_sketch_forward_noalloc(const void* X, const int64_t* offsets, int R,
                                         int64_t n_total, int d, const void* P, int k,
                                         const void* Wk, const void* Wv, sa_dtype dt,
                                         float* sketch, float* mass, float* lse,
                                         float* xsketch, int* device_status, void* stream) {
  // the forward runs without the helper grid when the scratch cannot hold its segments
  const size_t need = sa::forward_workspace_min(R, n_total, k, d, dt);
  // No plan for these arguments: the regular forward fails the same checks before any
  // launch (it never reads a workspace it was not given) and returns their exact code.
  if (need == 0)
    return sa_sketch_forward(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass, lse,
                             xsketch, nullptr, 0, stream);
  if (need > (size_t)SA_NOALLOC_SCRATCH_BYTES) return SA_ERR_WORKSPACE;
  void* scratch = nullptr;
  int st = scratch_for_current_device(&scratch);
  if (st != SA_OK) return st;
  st = sa_sketch_forward(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass, lse, xsketch,
                         scratch, (size_t)SA_NOALLOC_SCRATCH_BYTES, stream);
  if (st != SA_OK || device_status == nullptr) return st;
  const int dev_st = sa_sketch_get_device_status(scratch, stream);
  if (dev_st == SA_ERR_CUDA) return SA_ERR_CUDA;  // the status read itself failed
  *device_status = dev_st;
  return SA_OK;
}
