// C ABI of libsa_sketch.so: argument checks, the workspace plan, tensor maps and the
// launch sequence of Sketch Attention's forward and backward. See include/sa_sketch.h
// for the contract of every entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "sa_common.cuh"
#include "sa_internal.h"
#include "sa_sketch.h"

namespace sa {
namespace {

constexpr size_t kAlign = 256;
constexpr float kLog2e = 1.4426950408889634f;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Device {
  int id = -1;
  int sms = 0;
  bool ok = false;
};

sa_status current_device(Device* dev) {
  int id = 0;
  if (cudaGetDevice(&id) != cudaSuccess) return SA_ERR_NO_DEVICE;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, id) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, id) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, id) != cudaSuccess)
    return SA_ERR_NO_DEVICE;
  if (major != 10 || minor != 0) return SA_ERR_NO_DEVICE;  // built for sm_100a only
  dev->id = id;
  dev->sms = sms;
  dev->ok = true;
  return SA_OK;
}

// Co-resident clusters of the tcgen05 forward (which = 0) or of the single-pass backward
// (which = 1), cached per (device, kernel, d, C).
sa_status tc_clusters(const Device& dev, int d, int C, int* G, int which = 0) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev.id, which, d, C);
  auto it = cache.find(key);
  if (it == cache.end()) {
    int n = 0;
    const cudaError_t e =
        which == 0 ? fwd_sm100_max_clusters(d, C, &n) : bwd_fused_max_clusters(d, C, &n);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return SA_ERR_CUDA;
    }
    it = cache.emplace(key, n).first;
  }
  *G = it->second;
  return *G > 0 ? SA_OK : SA_ERR_UNSUPPORTED;
}

struct Plan {
  bool tc = false;  // tcgen05 path
  int C = 0, k_pad = 0, G = 0, Gb = 0;
  int H = 0, share = 0;  // forward helper CTAs and their share of the tiles (1/1024)
  size_t hdr = 0, ts = 0, pf = 0, pu = 0, pm = 0, lse2 = 0;
  size_t pn = 0, gt = 0, gh = 0, cj = 0, lseb = 0, db = 0, dppp = 0, dpp = 0, wvp = 0;
  // tensor-core finalize (bf16 forward, k a multiple of 128): U / mass as bf16 hi + lo
  bool ftc = false;
  size_t ubh = 0, ubl = 0;
  // tensor-core backward (bf16): the single-pass kernel's clusters in C and G
  bool btc = false;
  int wv_splits = 0;
  size_t ghb = 0, gtb = 0, gtlo = 0, ub = 0, pn2 = 0, pnn = 0, dpart = 0, lse2b = 0;
  size_t total = 0;
};

sa_status check_sizes(int R, int64_t n_total, int k, int d, sa_dtype dt) {
  if (R < 0 || R > SA_MAX_USERS || n_total < 0 || n_total > INT32_MAX) return SA_ERR_INVALID_ARG;
  if (dt != SA_F32 && dt != SA_BF16) return SA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
  if (k < 1 || k > SA_MAX_K) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

// helpers = false plans the bf16 forward without the helper grid (a smaller workspace:
// no helper segments).
sa_status make_plan(const Device& dev, int R, int64_t n_total, int k, int d, sa_dtype dt,
                    bool backward, Plan* p, bool helpers = true) {
  sa_status st = check_sizes(R, n_total, k, d, dt);
  if (st != SA_OK) return st;
  Plan q;
  q.tc = (dt == SA_BF16) && !backward;
  if (q.tc) {
    q.C = (k + 127) / 128;
    q.k_pad = q.C * 128;
    if ((st = tc_clusters(dev, d, q.C, &q.G)) != SA_OK) return st;
    if (helpers) fwd_sm100_helpers(d, q.C, q.G, dev.sms, &q.H, &q.share);
  } else {
    q.k_pad = (k + 31) / 32 * 32;
    const int pblocks = q.k_pad / 32;
    q.G = dev.sms * 4 / pblocks;
    if (q.G < 1) q.G = 1;
  }
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  q.hdr = take(sizeof(WsHeader));
  q.ts = take((size_t)(R + 1) * sizeof(long long));
  if (!backward) {
    q.pf = take((size_t)q.k_pad * d * (dt == SA_BF16 ? 2 : 4));
    const size_t segs = (size_t)q.G + (size_t)q.H + (size_t)R;
    q.pu = take(segs * q.k_pad * d * sizeof(float));
    q.pm = take(segs * q.k_pad * sizeof(float));
    if (!q.tc) q.lse2 = take((size_t)n_total * sizeof(float));
    if (q.tc && k == q.k_pad) {
      q.ftc = true;
      q.ubh = take((size_t)R * q.k_pad * d * 2);
      q.ubl = take((size_t)R * q.k_pad * d * 2);
    }
  } else if (dt == SA_BF16) {
    // tensor-core backward: the single-pass kernel keeps every token x prototype value
    // on chip; per-user Gh, Gt, c, per-cluster dPn partials, and the lse-recompute buffers
    q.btc = true;
    q.C = (k + 127) / 128;
    q.k_pad = q.C * 128;
    if ((st = tc_clusters(dev, d, q.C, &q.G, 1)) != SA_OK) return st;
    q.wv_splits = bwd_tc_wv_splits(dev.sms, R, q.k_pad);
    q.Gb = q.G;
    const size_t rkd = (size_t)R * q.k_pad * d;
    q.gt = take(rkd * sizeof(float));
    q.gtb = take(rkd * 2);
    q.gtlo = take(rkd * 2);
    q.ghb = take(rkd * 2);
    q.ub = take(rkd * 2);
    q.cj = take((size_t)R * q.k_pad * sizeof(float));
    q.pn2 = take((size_t)q.k_pad * d * 2);
    q.pnn = take((size_t)q.k_pad * d * 2);
    q.dpart = take((size_t)n_total * (q.k_pad / 64) * sizeof(float));
    q.lse2b = take((size_t)n_total * sizeof(float));
    q.dppp = take((size_t)q.G * q.k_pad * d * sizeof(float));
    q.dpp = take((size_t)q.k_pad * d * sizeof(float));
    q.wvp = take((size_t)(q.wv_splits > 1 ? q.wv_splits : 1) * d * d * sizeof(float));
  } else {
    q.Gb = q.G;
    q.pn = take((size_t)q.k_pad * d * sizeof(float));
    q.gt = take((size_t)R * q.k_pad * d * sizeof(float));
    q.gh = take((size_t)R * q.k_pad * d * sizeof(float));
    q.cj = take((size_t)R * q.k_pad * sizeof(float));
    q.lseb = take((size_t)n_total * sizeof(float));
    q.db = take((size_t)n_total * sizeof(float));
    q.dppp = take((size_t)q.Gb * q.k_pad * d * sizeof(float));
    q.dpp = take((size_t)q.k_pad * d * sizeof(float));
    q.wvp = take(bwd_wv_chunks(R, k) * d * d * sizeof(float));
  }
  q.total = o;
  *p = q;
  return SA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Row-major [rows, d] bf16 matrix, boxes of 128 rows x `box_cols` columns; the swizzle
// width equals the box row (64 columns: 128B swizzle, 16 columns: 32B swizzle).
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_cols) {
  auto fn = tmap_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, 128};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

cudaError_t prof_mark(cudaEvent_t ev, cudaStream_t s) {
  return ev ? cudaEventRecord(ev, s) : cudaSuccess;
}

sa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SA_OK;
  cudaGetLastError();
  return SA_ERR_CUDA;
}

}  // namespace
}  // namespace sa

namespace sa {
thread_local cudaEvent_t g_prof_start = nullptr;
thread_local cudaEvent_t g_prof_stop = nullptr;

cudaError_t prof_mark_start(cudaStream_t s) {
  return g_prof_start ? cudaEventRecord(g_prof_start, s) : cudaSuccess;
}
cudaError_t prof_mark_stop(cudaStream_t s) {
  return g_prof_stop ? cudaEventRecord(g_prof_stop, s) : cudaSuccess;
}

// The forward's smallest workspace: the plan without the helper grid.
size_t forward_workspace_min(int R, int64_t n_total, int k, int d, sa_dtype dt) {
  Device dev;
  if (current_device(&dev) != SA_OK) return 0;
  Plan p;
  if (make_plan(dev, R, n_total, k, d, dt, false, &p, false) != SA_OK) return 0;
  return p.total;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda needed).
PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}
}  // namespace sa

using namespace sa;

extern "C" {

size_t sa_sketch_workspace_size(int R, int64_t n_total, int k, int d, sa_dtype dt, int backward) {
  Device dev;
  if (current_device(&dev) != SA_OK) return 0;
  Plan p;
  if (make_plan(dev, R, n_total, k, d, dt, backward != 0, &p) != SA_OK) return 0;
  return p.total;
}

int sa_sketch_forward(const void* X, const int64_t* offsets, int R, int64_t n_total, int d,
                      const void* P, int k, const void* Wk, const void* Wv, sa_dtype dt,
                      float* sketch, float* mass, float* lse, float* xsketch, void* workspace,
                      size_t ws_bytes, void* stream_) {
  sa_status st = check_sizes(R, n_total, k, d, dt);
  if (st != SA_OK) return st;
  if (!offsets || !P || !Wk || !Wv || (n_total > 0 && !X) || (R > 0 && (!sketch || !mass)))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(P) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(sketch) ||
      !aligned16(mass) || !aligned16(lse) || !aligned16(xsketch) || !aligned16(offsets))
    return SA_ERR_INVALID_ARG;
  Device dev;
  if ((st = current_device(&dev)) != SA_OK) return st;
  Plan p;
  if ((st = make_plan(dev, R, n_total, k, d, dt, false, &p)) != SA_OK) return st;
  // a workspace too small for the helper grid's segments but large enough without them
  // runs the clustered grid alone
  if (ws_bytes < p.total && p.H > 0 &&
      (st = make_plan(dev, R, n_total, k, d, dt, false, &p, false)) != SA_OK)
    return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || ws_bytes < p.total)
    return SA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  WsHeader* hdr = at<WsHeader>(workspace, p.hdr);
  long long* ts = at<long long>(workspace, p.ts);
  float* pu = at<float>(workspace, p.pu);
  float* pm = at<float>(workspace, p.pm);

  if ((st = cuda_status(launch_schedule(offsets, R, n_total, hdr, ts, s))) != SA_OK) return st;
  const float scale = kLog2e / std::sqrt((float)d);
  if ((st = cuda_status(launch_fold(P, Wk, dt, k, p.k_pad, d, scale, at<void>(workspace, p.pf),
                                    p.tc, s))) != SA_OK)
    return st;
  if (n_total > 0) {
    if (p.tc) {
      CUtensorMap tx, tp;
      if (!make_tmap_bf16(&tx, X, (uint64_t)n_total, d, 64) ||
          !make_tmap_bf16(&tp, at<void>(workspace, p.pf), (uint64_t)p.k_pad, d, 64))
        return SA_ERR_CUDA;
      FwdSm100Args a;
      a.tmap_x = &tx;
      a.tmap_p = &tp;
      a.offsets = offsets;
      a.R = R;
      a.k_valid = k;
      a.C = p.C;
      a.k_pad = p.k_pad;
      a.d = d;
      a.G = p.G;
      a.H = p.H;
      a.share = p.share;
      a.hdr = hdr;
      a.tile_start = ts;
      a.part_u = pu;
      a.part_m = pm;
      a.lse = lse;
      a.budget = kDefaultWaitBudget;
      if ((st = cuda_status(prof_mark(g_prof_start, s))) != SA_OK) return st;
      if ((st = cuda_status(launch_fwd_sm100(a, s))) != SA_OK) return st;
      if ((st = cuda_status(prof_mark(g_prof_stop, s))) != SA_OK) return st;
    } else {
      FwdSimtArgs a;
      a.X = static_cast<const float*>(X);
      a.offsets = offsets;
      a.R = R;
      a.k = k;
      a.k_pad = p.k_pad;
      a.d = d;
      a.G = p.G;
      a.Pf = at<float>(workspace, p.pf);
      a.hdr = hdr;
      a.tile_start = ts;
      a.lse2 = at<float>(workspace, p.lse2);
      a.lse = lse;
      a.n_total = n_total;
      a.part_u = pu;
      a.part_m = pm;
      if ((st = cuda_status(prof_mark(g_prof_start, s))) != SA_OK) return st;
      if ((st = cuda_status(launch_fwd_simt(a, s))) != SA_OK) return st;
      if ((st = cuda_status(prof_mark(g_prof_stop, s))) != SA_OK) return st;
    }
  }
  FinalizeArgs f;
  f.hdr = hdr;
  f.tile_start = ts;
  f.part_u = pu;
  f.part_m = pm;
  f.Wv = Wv;
  f.dt = dt;
  f.R = R;
  f.k = k;
  f.k_pad = p.k_pad;
  f.d = d;
  f.G = p.G;
  f.H = p.H;
  f.share = p.share;
  f.mass_lanes = 1;
  f.sketch = sketch;
  f.mass = mass;
  f.xsketch = xsketch;
  f.ubar_hi = p.ftc ? at<__nv_bfloat16>(workspace, p.ubh) : nullptr;
  f.ubar_lo = p.ftc ? at<__nv_bfloat16>(workspace, p.ubl) : nullptr;
  return cuda_status(p.ftc ? launch_finalize_tc(f, s) : launch_finalize(f, s));
}

size_t sa_stca_workspace_size(int R, int64_t n_cand, int k, int d, int backward) {
  if (R < 0 || R > SA_MAX_USERS || n_cand < 0 || n_cand > INT32_MAX) return 0;
  if ((d != 64 && d != 128) || k < 1 || k > SA_MAX_K) return 0;
  Device dev;
  if (backward && current_device(&dev) != SA_OK) return 0;
  StcaPlan p;
  return stca_plan(R, n_cand, k, d, backward != 0, backward ? dev.sms : 0, &p);
}

int sa_stca_forward(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand, int d,
                    const float* S, int k, const void* Wq, const void* WK, const void* WV,
                    float* out, float* lse, void* workspace, size_t ws_bytes, void* stream_) {
  if (R < 0 || R > SA_MAX_USERS || n_cand < 0 || n_cand > INT32_MAX) return SA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || k < 1 || k > SA_MAX_K) return SA_ERR_UNSUPPORTED;
  if (!cand_offsets || !Wq || !WK || !WV || (n_cand > 0 && (!Q || !out)) || (R > 0 && !S))
    return SA_ERR_INVALID_ARG;
  if ((long long)R * ((k + 127) / 128 * 128) > INT32_MAX) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(cand_offsets) || !aligned16(S) || !aligned16(Wq) ||
      !aligned16(WK) || !aligned16(WV) || !aligned16(out) || !aligned16(lse))
    return SA_ERR_INVALID_ARG;
  Device dev;
  sa_status st;
  if ((st = current_device(&dev)) != SA_OK) return st;
  StcaArgs a;
  stca_plan(R, n_cand, k, d, false, 0, &a.plan);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      ws_bytes < a.plan.total)
    return SA_ERR_WORKSPACE;
  a.Q = Q;
  a.coff = cand_offsets;
  a.R = R;
  a.k = k;
  a.d = d;
  a.n_cand = n_cand;
  a.S = S;
  a.Wq = Wq;
  a.WK = WK;
  a.WV = WV;
  a.out = out;
  a.lse = lse;
  a.workspace = workspace;
  return cuda_status(launch_stca_forward(a, static_cast<cudaStream_t>(stream_)));
}

int sa_stca_backward(const void* Q, const int64_t* cand_offsets, const int64_t* cand_offsets_host,
                     int R, int64_t n_cand, int d, const float* S, int k, const void* Wq,
                     const void* WK, const void* WV, const float* dout, float* dQ, float* dS,
                     float* dWq, float* dWK, float* dWV, void* workspace, size_t ws_bytes,
                     void* stream_) {
  if (R < 0 || R > SA_MAX_USERS || n_cand < 0 || n_cand > INT32_MAX) return SA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || k < 1 || k > SA_MAX_K) return SA_ERR_UNSUPPORTED;
  if (!cand_offsets || !cand_offsets_host || !Wq || !WK || !WV || !dWq || !dWK || !dWV ||
      (n_cand > 0 && (!Q || !dout || !dQ)) || (R > 0 && (!S || !dS)))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(cand_offsets) || !aligned16(S) || !aligned16(Wq) ||
      !aligned16(WK) || !aligned16(WV) || !aligned16(dout) || !aligned16(dQ) || !aligned16(dS) ||
      !aligned16(dWq) || !aligned16(dWK) || !aligned16(dWV))
    return SA_ERR_INVALID_ARG;
  // the host offsets decide the per-user GEMMs: check them before anything is launched
  if (cand_offsets_host[0] != 0 || cand_offsets_host[R] != n_cand) return SA_ERR_BAD_OFFSETS;
  for (int u = 0; u < R; ++u)
    if (cand_offsets_host[u + 1] < cand_offsets_host[u]) return SA_ERR_BAD_OFFSETS;
  Device dev;
  sa_status st;
  if ((st = current_device(&dev)) != SA_OK) return st;
  StcaArgs a;
  stca_plan(R, n_cand, k, d, true, dev.sms, &a.plan);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      ws_bytes < a.plan.total)
    return SA_ERR_WORKSPACE;
  a.Q = Q;
  a.coff = cand_offsets;
  a.R = R;
  a.k = k;
  a.d = d;
  a.n_cand = n_cand;
  a.S = S;
  a.Wq = Wq;
  a.WK = WK;
  a.WV = WV;
  a.out = nullptr;
  a.lse = nullptr;
  a.workspace = workspace;
  StcaGrads g;
  g.dout = dout;
  g.dQ = dQ;
  g.dS = dS;
  g.dWq = dWq;
  g.dWK = dWK;
  g.dWV = dWV;
  return cuda_status(launch_stca_backward(a, g, dev.sms, static_cast<cudaStream_t>(stream_)));
}

namespace {

// Arguments shared by the ragged-key forward and backward (SA_OK or an argument code).
int check_keys_args(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand, int d,
                    const void* Kx, int64_t n_keys, const int64_t* key_begin,
                    const int64_t* key_end, const void* Wq, const void* WK, const void* WV) {
  if (R < 0 || R > SA_MAX_USERS || n_cand < 0 || n_cand > INT32_MAX || n_keys < 0 ||
      n_keys > INT32_MAX)
    return SA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
  if (!cand_offsets || !Wq || !WK || !WV || (n_cand > 0 && !Q) || (n_keys > 0 && !Kx) ||
      (R > 0 && (!key_begin || !key_end)))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(cand_offsets) || !aligned16(Kx) || !aligned16(Wq) ||
      !aligned16(WK) || !aligned16(WV) || (reinterpret_cast<uintptr_t>(key_begin) & 7u) ||
      (reinterpret_cast<uintptr_t>(key_end) & 7u))
    return SA_ERR_INVALID_ARG;
  return SA_OK;
}

}  // namespace

size_t sa_stca_keys_workspace_size(int R, int64_t n_cand, int d, int backward) {
  if (R < 0 || R > SA_MAX_USERS || n_cand < 0 || n_cand > INT32_MAX) return 0;
  if (d != 64 && d != 128) return 0;
  Device dev;
  if (backward && current_device(&dev) != SA_OK) return 0;
  StcaKeysPlan p;
  return stca_keys_plan(R, n_cand, d, backward != 0, backward ? dev.sms : 0, &p);
}

int sa_stca_keys_forward(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand, int d,
                         const void* Kx, int64_t n_keys, const int64_t* key_begin,
                         const int64_t* key_end, const void* Wq, const void* WK, const void* WV,
                         float* out, float* lse, void* workspace, size_t ws_bytes, void* stream_) {
  int st = check_keys_args(Q, cand_offsets, R, n_cand, d, Kx, n_keys, key_begin, key_end, Wq, WK,
                           WV);
  if (st != SA_OK) return st;
  if ((n_cand > 0 && !out) || !aligned16(out) || !aligned16(lse)) return SA_ERR_INVALID_ARG;
  Device dev;
  if ((st = current_device(&dev)) != SA_OK) return st;
  StcaKeysArgs a;
  stca_keys_plan(R, n_cand, d, false, 0, &a.plan);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      ws_bytes < a.plan.total)
    return SA_ERR_WORKSPACE;
  a.Q = Q;
  a.coff = cand_offsets;
  a.R = R;
  a.d = d;
  a.n_cand = n_cand;
  a.Kx = Kx;
  a.n_keys = n_keys;
  a.kb = key_begin;
  a.ke = key_end;
  a.Wq = Wq;
  a.WK = WK;
  a.WV = WV;
  a.out = out;
  a.lse = lse;
  a.workspace = workspace;
  return cuda_status(launch_stca_keys_forward(a, static_cast<cudaStream_t>(stream_)));
}

int sa_stca_keys_backward(const void* Q, const int64_t* cand_offsets, int R, int64_t n_cand,
                          int d, const void* Kx, int64_t n_keys, const int64_t* key_begin,
                          const int64_t* key_end, const void* Wq, const void* WK, const void* WV,
                          const float* dout, float* dQ, float* dKx, int accumulate, float* dWq,
                          float* dWK, float* dWV, void* workspace, size_t ws_bytes, void* stream_) {
  int st = check_keys_args(Q, cand_offsets, R, n_cand, d, Kx, n_keys, key_begin, key_end, Wq, WK,
                           WV);
  if (st != SA_OK) return st;
  if (!dWq || !dWK || !dWV || (n_cand > 0 && (!dout || !dQ)) || (n_keys > 0 && !dKx) ||
      !aligned16(dout) || !aligned16(dQ) || !aligned16(dKx) || !aligned16(dWq) ||
      !aligned16(dWK) || !aligned16(dWV))
    return SA_ERR_INVALID_ARG;
  Device dev;
  if ((st = current_device(&dev)) != SA_OK) return st;
  StcaKeysArgs a;
  stca_keys_plan(R, n_cand, d, true, dev.sms, &a.plan);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      ws_bytes < a.plan.total)
    return SA_ERR_WORKSPACE;
  a.Q = Q;
  a.coff = cand_offsets;
  a.R = R;
  a.d = d;
  a.n_cand = n_cand;
  a.Kx = Kx;
  a.n_keys = n_keys;
  a.kb = key_begin;
  a.ke = key_end;
  a.Wq = Wq;
  a.WK = WK;
  a.WV = WV;
  a.out = nullptr;
  a.lse = nullptr;
  a.workspace = workspace;
  StcaKeysGrads g;
  g.dout = dout;
  g.dQ = dQ;
  g.dKx = dKx;
  g.accumulate = accumulate != 0;
  g.dWq = dWq;
  g.dWK = dWK;
  g.dWV = dWV;
  return cuda_status(launch_stca_keys_backward(a, g, static_cast<cudaStream_t>(stream_)));
}

int sa_stca_recent_ranges(const int64_t* offsets, int R, int64_t L, int64_t* key_begin,
                          int64_t* key_end, void* stream_) {
  if (R < 0 || R > SA_MAX_USERS || L < 0) return SA_ERR_INVALID_ARG;
  if (R > 0 && (!offsets || !key_begin || !key_end)) return SA_ERR_INVALID_ARG;
  Device dev;
  int st;
  if ((st = current_device(&dev)) != SA_OK) return st;
  return cuda_status(launch_recent_ranges(offsets, R, L, key_begin, key_end,
                                          static_cast<cudaStream_t>(stream_)));
}

int sa_sketch_pack(const float* sketch, int64_t rows, int d, int format, void* codes,
                   float* scales, void* stream) {
  if (rows < 0 || (format != SA_CODEC_BF16 && format != SA_CODEC_FP8)) return SA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
  if (rows > 0 && (!sketch || !codes || (format == SA_CODEC_FP8 && !scales)))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(sketch) || !aligned16(codes) || !aligned16(scales)) return SA_ERR_INVALID_ARG;
  return cuda_status(
      launch_sketch_pack(sketch, rows, d, format, codes, scales, static_cast<cudaStream_t>(stream)));
}

int sa_sketch_unpack(const void* codes, const float* scales, int64_t rows, int d, int format,
                     float* sketch, void* stream) {
  if (rows < 0 || (format != SA_CODEC_BF16 && format != SA_CODEC_FP8)) return SA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
  if (rows > 0 && (!sketch || !codes || (format == SA_CODEC_FP8 && !scales)))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(sketch) || !aligned16(codes) || !aligned16(scales)) return SA_ERR_INVALID_ARG;
  return cuda_status(launch_sketch_unpack(codes, scales, rows, d, format, sketch,
                                          static_cast<cudaStream_t>(stream)));
}

int sa_sketch_backward(const void* X, const int64_t* offsets, int R, int64_t n_total, int d,
                       const void* P, int k, const void* Wk, const void* Wv, sa_dtype dt,
                       const float* sketch, const float* mass, const float* lse,
                       const float* xsketch, const float* dsketch, const float* dmass, float* dX,
                       float* dP, float* dWk, float* dWv, void* workspace, size_t ws_bytes,
                       void* stream_) {
  sa_status st = check_sizes(R, n_total, k, d, dt);
  if (st != SA_OK) return st;
  if (!offsets || !P || !Wk || !Wv || !dP || !dWk || !dWv ||
      (n_total > 0 && (!X || !dX)) ||
      (R > 0 && (!sketch || !mass || !xsketch || !dsketch)))
    return SA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(P) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(sketch) ||
      !aligned16(mass) || !aligned16(xsketch) || !aligned16(dsketch) || !aligned16(dmass) ||
      !aligned16(dX) || !aligned16(dP) || !aligned16(dWk) || !aligned16(dWv) || !aligned16(offsets) ||
      !aligned16(lse))
    return SA_ERR_INVALID_ARG;
  Device dev;
  if ((st = current_device(&dev)) != SA_OK) return st;
  Plan p;
  if ((st = make_plan(dev, R, n_total, k, d, dt, true, &p)) != SA_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || ws_bytes < p.total)
    return SA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  WsHeader* hdr = at<WsHeader>(workspace, p.hdr);
  long long* ts = at<long long>(workspace, p.ts);
  if ((st = cuda_status(launch_schedule(offsets, R, n_total, hdr, ts, s))) != SA_OK) return st;
  if (!p.btc &&
      (st = cuda_status(launch_fold(P, Wk, dt, k, p.k_pad, d, 1.0f / std::sqrt((float)d),
                                    at<void>(workspace, p.pn), false, s))) != SA_OK)
    return st;
  BwdArgs a = {};
  a.X = X;
  a.dt = dt;
  a.offsets = offsets;
  a.R = R;
  a.k = k;
  a.k_pad = p.k_pad;
  a.d = d;
  a.G = p.Gb;
  a.n_total = n_total;
  a.P = P;
  a.Wk = Wk;
  a.Wv = Wv;
  a.sketch = sketch;
  a.mass = mass;
  a.xsketch = xsketch;
  a.dsketch = dsketch;
  a.dmass = dmass;
  a.hdr = hdr;
  a.tile_start = ts;
  a.Pn = at<float>(workspace, p.pn);
  a.Gt = at<float>(workspace, p.gt);
  a.Gh = at<float>(workspace, p.gh);
  a.cj = at<float>(workspace, p.cj);
  a.lseb = at<float>(workspace, p.lseb);
  a.Db = at<float>(workspace, p.db);
  a.dpp_part = at<float>(workspace, p.dppp);
  a.dpp = at<float>(workspace, p.dpp);
  a.wv_part = at<float>(workspace, p.wvp);
  a.dX = dX;
  a.dP = dP;
  a.dWk = dWk;
  a.dWv = dWv;
  if (!p.btc) return cuda_status(launch_bwd_simt(a, s));
  // bf16: tensor-core backward (the SIMT-only buffers are unused)
  a.Pn = nullptr;
  a.Gh = nullptr;
  a.Ghb = at<__nv_bfloat16>(workspace, p.ghb);
  a.Gtb = at<__nv_bfloat16>(workspace, p.gtb);
  a.Gtlo = at<__nv_bfloat16>(workspace, p.gtlo);
  a.lseb = nullptr;
  a.Db = nullptr;
  BwdTcArgs t;
  t.b = a;
  t.lse = lse;
  t.pn2 = at<__nv_bfloat16>(workspace, p.pn2);
  t.pnn = at<__nv_bfloat16>(workspace, p.pnn);
  t.dpart = at<float>(workspace, p.dpart);
  t.lse2 = at<float>(workspace, p.lse2b);
  t.Ub = at<__nv_bfloat16>(workspace, p.ub);
  t.C = p.C;
  t.G = p.G;
  t.wv_splits = p.wv_splits;
  return cuda_status(launch_bwd_tc(t, s));
}

int sa_sketch_combine(const float* xsketch, const float* mass, int R, int k, int d, const void* Wv,
                      sa_dtype dt, float* sketch, void* stream_) {
  if (R < 0 || R > SA_MAX_USERS || k < 1 || k > SA_MAX_K) return SA_ERR_INVALID_ARG;
  if (dt != SA_F32 && dt != SA_BF16) return SA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SA_ERR_UNSUPPORTED;
  if (R == 0) return SA_OK;
  if (!xsketch || !mass || !Wv || !sketch) return SA_ERR_INVALID_ARG;
  if (!aligned16(xsketch) || !aligned16(mass) || !aligned16(Wv) || !aligned16(sketch))
    return SA_ERR_INVALID_ARG;
  Device dev;
  sa_status st = current_device(&dev);
  if (st != SA_OK) return st;
  return cuda_status(launch_combine(xsketch, mass, R, k, d, Wv, dt, sketch,
                                    static_cast<cudaStream_t>(stream_)));
}

int sa_sketch_debug_gemm(const void* A, int a_mn, const void* B, int b_mn, int M, int N, int K,
                         int splits, float* out, void* workspace, void* stream_) {
  if (!A || !B || !out || !workspace || M < 1 || N < 1 || K < 1 || splits < 1 ||
      splits > (K + 63) / 64 || (N % 4) != 0)
    return SA_ERR_INVALID_ARG;
  if (((a_mn ? M : K) % 8) != 0 || ((b_mn ? N : K) % 8) != 0) return SA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || !aligned16(A) || !aligned16(B) ||
      !aligned16(out))
    return SA_ERR_INVALID_ARG;
  Device dev;
  sa_status st = current_device(&dev);
  if (st != SA_OK) return st;
  GemmArgs g = {};
  g.a[0] = {A, (uint64_t)(a_mn ? K : M), (uint64_t)(a_mn ? M : K), a_mn != 0};
  g.b[0] = {B, (uint64_t)(b_mn ? K : N), (uint64_t)(b_mn ? N : K), b_mn != 0};
  g.phases = 1;
  g.k_tiles[0] = (K + 63) / 64;
  g.M = M;
  g.N = N;
  g.m_tiles_bound = (M + 127) / 128;
  g.splits = splits;
  g.epi = kEpiStoreF32;
  g.hdr = static_cast<const WsHeader*>(workspace);
  g.out_f32 = out;
  g.ld_out = N;
  g.split_stride = (long long)M * N;
  return cuda_status(launch_gemm(g, static_cast<cudaStream_t>(stream_)));
}

int sa_sketch_forward_grid(int k, int d, sa_dtype dt, int* clusters, int* cluster_size,
                           int* helpers, int* helper_share) {
  if (!clusters || !cluster_size) return SA_ERR_INVALID_ARG;
  sa_status st = check_sizes(0, 0, k, d, dt);
  if (st != SA_OK) return st;
  Device dev;
  if ((st = current_device(&dev)) != SA_OK) return st;
  Plan p;
  if ((st = make_plan(dev, 0, 0, k, d, dt, false, &p)) != SA_OK) return st;
  *clusters = p.tc ? p.G : 0;
  *cluster_size = p.tc ? p.C : 0;
  if (helpers) *helpers = p.tc ? p.H : 0;
  if (helper_share) *helper_share = p.tc ? p.share : 0;
  return SA_OK;
}

int sa_sketch_get_device_status(const void* workspace, void* stream_) {
  if (!workspace) return SA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  int h = 0;
  if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return SA_ERR_CUDA;
  }
  return h;
}

int sa_sketch_profile_events(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr)) return SA_ERR_INVALID_ARG;
  g_prof_start = static_cast<cudaEvent_t>(start_event);
  g_prof_stop = static_cast<cudaEvent_t>(stop_event);
  return SA_OK;
}

const char* sa_status_string(int status) {
  switch (status) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG: null, negative or misaligned argument";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED: shape outside the implemented range";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE: workspace null, misaligned or too small";
    case SA_ERR_CUDA: return "SA_ERR_CUDA: a CUDA call failed";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    case SA_ERR_BAD_OFFSETS: return "SA_ERR_BAD_OFFSETS: offsets are not a ragged partition";
    case SA_ERR_NO_DEVICE: return "SA_ERR_NO_DEVICE: no sm_100 device is current";
    default: return "unknown sa_status";
  }
}

int sa_sketch_debug_wait_timeout(void* workspace, long long budget_cycles, void* stream_) {
  if (!workspace || budget_cycles <= 0) return SA_ERR_INVALID_ARG;
  Device dev;
  sa_status st = current_device(&dev);
  if (st != SA_OK) return st;
  return cuda_status(launch_debug_wait_timeout(static_cast<WsHeader*>(workspace), budget_cycles,
                                               static_cast<cudaStream_t>(stream_)));
}

}  // extern "C"
