// Small kernels around the hot loop: the ragged-batch schedule, the prototype fold,
// the split-n finalize, and the failure-detection test hook.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

// ------------------------------------------------------------------ schedule
// One block. Clears the status word, checks that offsets describe a ragged partition
// of [0, n_total) (offsets[0] = 0, non-decreasing, offsets[R] = n_total), and writes the
// exclusive prefix sum of per-user tile counts, tile_start[0..R], tile = 128 tokens.
__global__ void __launch_bounds__(1024) schedule_kernel(const int64_t* __restrict__ off, int R,
                                                        int64_t n_total, WsHeader* hdr,
                                                        long long* __restrict__ ts) {
  __shared__ long long part[1024];
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) {
    hdr->status = 0;
    bad = (off[0] != 0 || off[R] != n_total) ? 1 : 0;
  }
  __syncthreads();
  const int chunk = (R + 1023) / 1024;
  const int u0 = min(R, tid * chunk), u1 = min(R, u0 + chunk);
  long long local = 0;
  int my_bad = 0;
  for (int u = u0; u < u1; ++u) {
    const long long n = off[u + 1] - off[u];
    if (n < 0) my_bad = 1;
    else local += (n + kTileTokens - 1) / kTileTokens;
  }
  if (my_bad) bad = 1;
  part[tid] = local;
  __syncthreads();
  if (tid == 0) {
    long long acc = 0;
    for (int i = 0; i < 1024; ++i) {
      const long long v = part[i];
      part[i] = acc;
      acc += v;
    }
    if (bad) {
      hdr->total_tiles = 0;
      hdr->status = SA_ERR_BAD_OFFSETS;
    } else {
      hdr->total_tiles = acc;
    }
    ts[R] = acc;
  }
  __syncthreads();
  long long run = part[tid];
  for (int u = u0; u < u1; ++u) {
    ts[u] = run;
    const long long n = off[u + 1] - off[u];
    if (n > 0) run += (n + kTileTokens - 1) / kTileTokens;
  }
}

// ------------------------------------------------------------------ fold
// Pf[j][c] = scale * sum_e P[j][e] Wk[c][e]   (so P_j . (X_t Wk) = X_t . Pf_j / scale).
// Block: 32 prototypes x all d outputs; Wk staged transposed-free with a padded stride.
template <typename TIn>
__device__ __forceinline__ float to_f(TIn v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename TIn>
__global__ void __launch_bounds__(256) fold_kernel(const TIn* __restrict__ P, const TIn* __restrict__ Wk,
                                                   int k, int k_pad, int d, float scale,
                                                   void* __restrict__ out, int out_bf16) {
  extern __shared__ float fsm[];
  float* wk = fsm;                      // [d][d+1]
  float* ps = fsm + d * (d + 1);        // [32][d]
  const int j0 = blockIdx.x * 32;
  for (int i = threadIdx.x; i < d * d; i += blockDim.x) {
    const int c = i / d, e = i % d;
    wk[c * (d + 1) + e] = to_f(Wk[i]);
  }
  for (int i = threadIdx.x; i < 32 * d; i += blockDim.x) {
    const int jj = i / d, e = i % d;
    ps[i] = (j0 + jj < k) ? to_f(P[(size_t)(j0 + jj) * d + e]) : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * d; i += blockDim.x) {
    const int jj = i / d, c = i % d;
    float acc = 0.f;
    for (int e = 0; e < d; ++e) acc = fmaf(ps[jj * d + e], wk[c * (d + 1) + e], acc);
    acc *= scale;
    const size_t o = (size_t)(j0 + jj) * d + c;
    if (j0 + jj < k_pad) {
      if (out_bf16) reinterpret_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(acc);
      else reinterpret_cast<float*>(out)[o] = acc;
    }
  }
}

// ------------------------------------------------------------------ finalize
// Block (user u, 32 prototypes). The user's segments are the clusters whose tile range
// intersects the user's tiles; their partials are added in cluster order, so the
// result does not depend on timing. Then sketch_j = (U_j Wv) / mass_j, mass_j = 0 -> 0.
__device__ __forceinline__ long long range_start(long long g, long long T, int G) {
  return g * T / G;
}

__device__ int cluster_of_tile(long long x, long long T, int G) {
  long long g = x * G / T;
  if (g >= G) g = G - 1;
  while (g + 1 < G && range_start(g + 1, T, G) <= x) ++g;
  while (g > 0 && range_start(g, T, G) > x) --g;
  return (int)g;
}

template <typename TIn>
__global__ void __launch_bounds__(256) finalize_kernel(FinalizeArgs a, const TIn* __restrict__ Wv) {
  extern __shared__ float fsm[];
  const int d = a.d;
  float* wv = fsm;              // [d][d]
  float* us = fsm + d * d;      // [32][d]
  float* ms = us + 32 * d;      // [32]
  const int u = blockIdx.x;
  const int j0 = blockIdx.y * 32;
  if (read_status(&a.hdr->status) != 0) return;
  const long long T = a.hdr->total_tiles;
  const long long x0 = a.tile_start[u], x1 = a.tile_start[u + 1];
  for (int i = threadIdx.x; i < 32 * d; i += blockDim.x) us[i] = 0.f;
  if (threadIdx.x < 32) ms[threadIdx.x] = 0.f;
  __syncthreads();
  if (x1 > x0) {
    const int g0 = cluster_of_tile(x0, T, a.G), g1 = cluster_of_tile(x1 - 1, T, a.G);
    for (int g = g0; g <= g1; ++g) {
      if (range_start(g, T, a.G) == range_start(g + 1, T, a.G)) continue;  // empty range
      const size_t seg = (size_t)g + u;
      const float* src = a.part_u + (seg * a.k_pad + j0) * d;
      for (int i = threadIdx.x; i < 32 * d; i += blockDim.x) us[i] += src[i];
      if (threadIdx.x < 32) {
        const float* pm = a.part_m + (seg * a.k_pad + j0 + threadIdx.x) * a.mass_lanes;
        float v = 0.f;
        for (int l = 0; l < a.mass_lanes; ++l) v += pm[l];
        ms[threadIdx.x] += v;
      }
    }
  }
  for (int i = threadIdx.x; i < d * d; i += blockDim.x) wv[i] = to_f(Wv[i]);
  __syncthreads();
  // outputs
  for (int i = threadIdx.x; i < 32 * d; i += blockDim.x) {
    const int jj = i / d, e = i % d;
    if (j0 + jj < a.k && a.xsketch) a.xsketch[((size_t)u * a.k + j0 + jj) * d + e] = us[i];
  }
  if (threadIdx.x < 32 && j0 + threadIdx.x < a.k) a.mass[(size_t)u * a.k + j0 + threadIdx.x] = ms[threadIdx.x];
  const int e = threadIdx.x % d;
  const int jstep = blockDim.x / d;
  for (int jj = threadIdx.x / d; jj < 32; jj += jstep) {
    if (j0 + jj >= a.k) break;
    float acc = 0.f;
    for (int c = 0; c < d; ++c) acc = fmaf(us[jj * d + c], wv[c * d + e], acc);
    const float m = ms[jj];
    a.sketch[((size_t)u * a.k + j0 + jj) * d + e] = m > 0.f ? acc / m : 0.f;
  }
}

// ------------------------------------------------------------------ test hook
__global__ void debug_wait_timeout_kernel(WsHeader* hdr, long long budget) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x == 0) {
    hdr->status = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the bounded wait must give up and latch the timeout
    mbar_wait(smem_u32(&bar), 0, &hdr->status, budget);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_schedule(const int64_t* offsets, int R, int64_t n_total, WsHeader* hdr,
                            long long* tile_start, cudaStream_t s) {
  schedule_kernel<<<1, 1024, 0, s>>>(offsets, R, n_total, hdr, tile_start);
  return cudaGetLastError();
}

cudaError_t launch_fold(const void* P, const void* Wk, sa_dtype dt, int k, int k_pad, int d,
                        float scale, void* Pf, bool out_bf16, cudaStream_t s) {
  const size_t smem = (size_t)(d * (d + 1) + 32 * d) * sizeof(float);
  const dim3 grid((unsigned)((k_pad + 31) / 32));
  cudaError_t e;
  if (dt == SA_BF16) {
    e = cudaFuncSetAttribute(fold_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fold_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(
        static_cast<const __nv_bfloat16*>(P), static_cast<const __nv_bfloat16*>(Wk), k, k_pad, d,
        scale, Pf, out_bf16 ? 1 : 0);
  } else {
    e = cudaFuncSetAttribute(fold_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fold_kernel<float><<<grid, 256, smem, s>>>(static_cast<const float*>(P),
                                               static_cast<const float*>(Wk), k, k_pad, d, scale,
                                               Pf, out_bf16 ? 1 : 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t s) {
  if (a.R == 0) return cudaSuccess;
  const size_t smem = (size_t)(a.d * a.d + 32 * a.d + 32) * sizeof(float);
  const dim3 grid((unsigned)a.R, (unsigned)((a.k + 31) / 32));
  cudaError_t e;
  if (a.dt == SA_BF16) {
    e = cudaFuncSetAttribute(finalize_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    finalize_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(a, static_cast<const __nv_bfloat16*>(a.Wv));
  } else {
    e = cudaFuncSetAttribute(finalize_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    finalize_kernel<float><<<grid, 256, smem, s>>>(a, static_cast<const float*>(a.Wv));
  }
  return cudaGetLastError();
}

cudaError_t launch_debug_wait_timeout(WsHeader* hdr, long long budget, cudaStream_t s) {
  debug_wait_timeout_kernel<<<1, 32, 0, s>>>(hdr, budget);
  return cudaGetLastError();
}

}  // namespace sa
