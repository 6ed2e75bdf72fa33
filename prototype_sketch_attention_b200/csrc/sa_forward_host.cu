// sa_sketch_forward_host: the Sketch Attention forward from host memory to host memory.
//
// The history tokens of a ragged batch usually start on the host (a feature store, a
// data loader). Copying all of X before the forward starts leaves the GPU idle for the
// whole copy, and at 2 d bytes per token the copy is far longer than the forward (the
// forward reads X once at HBM speed; the host link is two orders of magnitude slower).
// This entry point cuts the users into parts of about equal token count and pipelines
// them over three streams: part p's X goes to the device on the copy-in stream while
// part p - 1's forward runs on the compute stream, and part p's sketch and mass go back
// on the copy-out stream as soon as its forward is done. Users are independent in the
// forward (the blog's "3. The system makes it cheap enough to matter": multi-request
// batching groups independent users), so a part is one ordinary forward call and nothing
// has to be combined afterwards.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "sa_sketch.h"

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

constexpr int kMaxParts = 64;

// Part table, passed by value to the rebase kernel (no host staging buffer to copy).
struct Parts {
  int np;
  int bounds[kMaxParts + 1];  // part p holds users [bounds[p], bounds[p + 1])
  int slot[kMaxParts];        // first entry of part p's rebased offsets (an even index)
};

// Rebased offsets of every part, side by side: part p's R_p + 1 entries start at
// slot[p] (an even index, so each part's array is 16-byte aligned) and hold
// offsets[u0 + i] - offsets[u0].
__global__ void rebase_offsets_kernel(const int64_t* __restrict__ off, const Parts parts,
                                      int64_t* __restrict__ out) {
  for (int p = 0; p < parts.np; ++p) {
    const int u0 = parts.bounds[p], u1 = parts.bounds[p + 1];
    const int64_t base = off[u0];
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= u1 - u0; i += gridDim.x * blockDim.x)
      out[parts.slot[p] + i] = off[u0 + i] - base;
  }
}

struct Layout {
  size_t x = 0, off = 0, roff = 0, sketch = 0, mass = 0, ws = 0, ws_bytes = 0, total = 0;
};

size_t elem_bytes(sa_dtype dt) { return dt == SA_BF16 ? 2 : 4; }

// Device buffer layout for these sizes (ws_bytes from sa_sketch_workspace_size).
bool make_layout(int R, int64_t n_total, int k, int d, sa_dtype dt, int parts, Layout* L) {
  const size_t ws = sa_sketch_workspace_size(R, n_total, k, d, dt, 0);
  if (ws == 0) return false;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L->x = take((size_t)n_total * d * elem_bytes(dt));
  L->off = take((size_t)(R + 1) * sizeof(int64_t));
  L->roff = take((size_t)(R + 2 * parts + 2) * sizeof(int64_t));
  L->sketch = take((size_t)R * k * d * sizeof(float));
  L->mass = take((size_t)R * k * sizeof(float));
  L->ws = take(ws);
  L->ws_bytes = ws;
  L->total = o;
  return true;
}

int cuda_fail() {
  cudaGetLastError();
  return SA_ERR_CUDA;
}

}  // namespace

extern "C" {

int sa_sketch_host_parts(const int64_t* offsets_host, int R, int parts, int* bounds) {
  if (!offsets_host || !bounds || R < 0 || parts < 1) return -SA_ERR_INVALID_ARG;
  if (R == 0) return 0;
  const int64_t n_total = offsets_host[R];
  if (offsets_host[0] != 0 || n_total < 0) return -SA_ERR_INVALID_ARG;
  for (int u = 0; u < R; ++u)
    if (offsets_host[u + 1] < offsets_host[u]) return -SA_ERR_INVALID_ARG;
  // cut c ends the part at the first user whose tokens reach c / parts of the total; a
  // cut that gives an empty part (no new user, or no new tokens) is dropped, and users
  // without tokens at the end join the last part
  int np = 0;
  bounds[np++] = 0;
  for (int c = 1; c < parts; ++c) {
    const int64_t target = n_total * c / parts;
    int lo = 0, hi = R;  // first u in [0, R) with offsets[u + 1] >= target
    while (lo < hi) {
      const int mid = (lo + hi) / 2;
      if (offsets_host[mid + 1] >= target) hi = mid; else lo = mid + 1;
    }
    const int u1 = lo + 1;
    if (u1 > 0 && u1 < R && u1 > bounds[np - 1] && offsets_host[u1] > offsets_host[bounds[np - 1]])
      bounds[np++] = u1;
  }
  while (np > 1 && offsets_host[bounds[np - 1]] == n_total) --np;
  bounds[np] = R;
  return np;
}

size_t sa_sketch_forward_host_buffer_size(int R, int64_t n_total, int k, int d, sa_dtype dt,
                                          int parts) {
  if (parts < 1) return 0;
  Layout L;
  return make_layout(R, n_total, k, d, dt, parts, &L) ? L.total : 0;
}

int sa_sketch_forward_host_status(const void* device_buffer, int R, int64_t n_total, int k,
                                  int d, sa_dtype dt, int parts, void* stream) {
  if (!device_buffer || parts < 1 || parts > kMaxParts) return SA_ERR_INVALID_ARG;
  if (k % 4 != 0) parts = 1;
  Layout L;
  if (!make_layout(R, n_total, k, d, dt, parts, &L)) return SA_ERR_INVALID_ARG;
  return sa_sketch_get_device_status(static_cast<const uint8_t*>(device_buffer) + L.ws, stream);
}

int sa_sketch_forward_host(const void* X_host, const int64_t* offsets_host, int R, int64_t n_total,
                           int d, const void* P, int k, const void* Wk, const void* Wv, sa_dtype dt,
                           float* sketch_host, float* mass_host, void* device_buffer,
                           size_t device_bytes, int parts, void* stream, void* h2d_stream,
                           void* d2h_stream) {
  if (!offsets_host || R < 0 || R > SA_MAX_USERS || n_total < 0 || parts < 1 || parts > kMaxParts)
    return SA_ERR_INVALID_ARG;
  if ((n_total > 0 && !X_host) || (R > 0 && (!sketch_host || !mass_host)) || !P || !Wk || !Wv)
    return SA_ERR_INVALID_ARG;
  if (dt != SA_F32 && dt != SA_BF16) return SA_ERR_INVALID_ARG;
  if (offsets_host[0] != 0 || offsets_host[R] != n_total) return SA_ERR_BAD_OFFSETS;
  for (int u = 0; u < R; ++u)
    if (offsets_host[u + 1] < offsets_host[u]) return SA_ERR_BAD_OFFSETS;
  if (k % 4 != 0) parts = 1;  // every part's mass rows must start 16-byte aligned
  Layout L;
  if (!make_layout(R, n_total, k, d, dt, parts, &L)) {
    // no plan: the regular forward reports the exact argument code before any launch
    const int st = sa_sketch_forward(X_host, offsets_host, R, n_total, d, P, k, Wk, Wv, dt,
                                     sketch_host, mass_host, nullptr, nullptr, nullptr, 0, stream);
    return st != SA_OK ? st : SA_ERR_UNSUPPORTED;
  }
  if (!device_buffer || (reinterpret_cast<uintptr_t>(device_buffer) % kAlign) != 0 ||
      device_bytes < L.total)
    return SA_ERR_WORKSPACE;
  if (R == 0) return SA_OK;

  Parts pt = {};
  pt.np = sa_sketch_host_parts(offsets_host, R, parts, pt.bounds);
  if (pt.np < 1) return SA_ERR_BAD_OFFSETS;
  const int np = pt.np;
  for (int p = 0, at = 0; p < np; ++p) {
    pt.slot[p] = at;
    at += ((pt.bounds[p + 1] - pt.bounds[p]) + 2) & ~1;
  }

  uint8_t* base = static_cast<uint8_t*>(device_buffer);
  uint8_t* Xd = base + L.x;
  int64_t* offd = reinterpret_cast<int64_t*>(base + L.off);
  int64_t* roff = reinterpret_cast<int64_t*>(base + L.roff);
  float* sk = reinterpret_cast<float*>(base + L.sketch);
  float* ms = reinterpret_cast<float*>(base + L.mass);
  void* ws = base + L.ws;
  const size_t xrow = (size_t)d * elem_bytes(dt);

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaStream_t hs = static_cast<cudaStream_t>(h2d_stream);
  cudaStream_t ds = static_cast<cudaStream_t>(d2h_stream);
  // Events order the three streams; they are released as soon as the work that records
  // them has run (cudaEventDestroy does not wait), so nothing outlives the call.
  std::vector<cudaEvent_t> ev;
  auto new_event = [&](cudaEvent_t* e) {
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
    ev.push_back(*e);
    return true;
  };
  auto release = [&]() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  };
  int st = SA_OK;
  do {
    // the copy streams start after the work already queued on the compute stream (an
    // earlier call may still be reading the same device buffer)
    cudaEvent_t start;
    if (!new_event(&start) || cudaEventRecord(start, cs) != cudaSuccess ||
        cudaStreamWaitEvent(hs, start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(ds, start, 0) != cudaSuccess) {
      st = cuda_fail();
      break;
    }
    // offsets first (small), then the rebased offsets of every part
    if (cudaMemcpyAsync(offd, offsets_host, (size_t)(R + 1) * sizeof(int64_t),
                        cudaMemcpyHostToDevice, hs) != cudaSuccess) {
      st = cuda_fail();
      break;
    }
    rebase_offsets_kernel<<<(R + 256) / 256 < 64 ? (R + 256) / 256 : 64, 256, 0, hs>>>(offd, pt,
                                                                                       roff);
    if (cudaGetLastError() != cudaSuccess) {
      st = SA_ERR_CUDA;
      break;
    }
    for (int p = 0; p < np && st == SA_OK; ++p) {
      const int u0 = pt.bounds[p], u1 = pt.bounds[p + 1];
      const int64_t t0 = offsets_host[u0], t1 = offsets_host[u1];
      cudaEvent_t landed, done;
      if (t1 > t0 &&
          cudaMemcpyAsync(Xd + (size_t)t0 * xrow, static_cast<const uint8_t*>(X_host) + (size_t)t0 * xrow,
                          (size_t)(t1 - t0) * xrow, cudaMemcpyHostToDevice, hs) != cudaSuccess) {
        st = cuda_fail();
        break;
      }
      if (!new_event(&landed) || cudaEventRecord(landed, hs) != cudaSuccess ||
          cudaStreamWaitEvent(cs, landed, 0) != cudaSuccess) {
        st = cuda_fail();
        break;
      }
      st = sa_sketch_forward(Xd + (size_t)t0 * xrow, roff + pt.slot[p], u1 - u0, t1 - t0, d, P, k, Wk,
                             Wv, dt, sk + (size_t)u0 * k * d, ms + (size_t)u0 * k, nullptr, nullptr,
                             ws, L.ws_bytes, cs);
      if (st != SA_OK) break;
      if (!new_event(&done) || cudaEventRecord(done, cs) != cudaSuccess ||
          cudaStreamWaitEvent(ds, done, 0) != cudaSuccess ||
          cudaMemcpyAsync(sketch_host + (size_t)u0 * k * d, sk + (size_t)u0 * k * d,
                          (size_t)(u1 - u0) * k * d * sizeof(float), cudaMemcpyDeviceToHost,
                          ds) != cudaSuccess ||
          cudaMemcpyAsync(mass_host + (size_t)u0 * k, ms + (size_t)u0 * k,
                          (size_t)(u1 - u0) * k * sizeof(float), cudaMemcpyDeviceToHost,
                          ds) != cudaSuccess) {
        st = cuda_fail();
        break;
      }
    }
    if (st != SA_OK) break;
    // the compute stream ends after the last copy back: synchronising it (or an event
    // recorded on it) makes the host outputs visible
    cudaEvent_t back;
    if (!new_event(&back) || cudaEventRecord(back, ds) != cudaSuccess ||
        cudaStreamWaitEvent(cs, back, 0) != cudaSuccess)
      st = cuda_fail();
  } while (false);
  release();
  return st;
}

}  // extern "C"
