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
  __shared__ long long part[64];
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
  // exclusive prefix sum of the per-thread tile counts: warp scans, then the warp totals
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((tid & 31) >= o) incl += v;
  }
  if ((tid & 31) == 31) part[tid >> 5] = incl;
  __syncthreads();
  if (tid < 32) {
    long long w = part[tid];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, w, o);
      if (tid >= o) w += v;
    }
    part[32 + tid] = w;  // inclusive scan of the warp totals
  }
  __syncthreads();
  const long long base = (tid >= 32 ? part[32 + (tid >> 5) - 1] : 0) + incl - local;
  if (tid == 1023) {
    const long long acc = part[32 + 31];
    if (bad) {
      hdr->total_tiles = 0;
      hdr->status = SA_ERR_BAD_OFFSETS;
    } else {
      hdr->total_tiles = acc;
    }
    ts[R] = acc;
  }
  long long run = base;
  for (int u = u0; u < u1; ++u) {
    ts[u] = run;
    const long long n = off[u + 1] - off[u];
    if (n > 0) run += (n + kTileTokens - 1) / kTileTokens;
  }
}

// ------------------------------------------------------------------ fold (helpers)
// Pf[j][c] = scale * sum_e P[j][e] Wk[c][e]   (so P_j . (X_t Wk) = X_t . Pf_j / scale).
template <typename TIn>
__device__ __forceinline__ float to_f(TIn v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// ------------------------------------------------------------------ finalize (helpers)
// A user's segments are the tile ranges (TileRanges: clusters, then helper CTAs) that
// intersect the user's tiles; their partials are added in range order, so the result does
// not depend on timing. Then sketch_j = (U_j Wv) / mass_j, with mass_j = 0 -> 0.

// ------------------------------------------------------------------ tiled row GEMM
// out[j][e] = sum_c lr[j][c] * rm[c][e] for a tile of 64 rows j and D columns e, both
// operands in shared memory with row stride D+4 floats. 256 threads: kTE = D/4 threads
// across e (4 columns each) and 256/kTE across rows, kJPT rows each. Per 4 values of c a
// thread reads kJPT float4 of lr (the same address across a warp's e lanes) and 4 float4
// of rm, then issues 16*kJPT FMAs.
constexpr int kRowTile = 64;      // finalize / combine: rows per block
constexpr int kFoldRowTile = 16;  // fold: rows per block (k / 16 blocks)

template <int D, int RT = kRowTile>
struct TileShape {
  static constexpr int kLd = D + 4;
  static constexpr int kTE = D / 4;
  static constexpr int kTJ = 256 / kTE;
  static constexpr int kJPT = RT / kTJ;
  static_assert(kJPT >= 1, "row tile");
};

// rm[c][e] = W[c * D + e] (transpose = false) or W[e * D + c] (true), row stride D + 4,
// from 16-byte loads of W (8 bf16 or 4 fp32 consecutive elements).
template <int D, typename TIn, bool kTranspose>
__device__ __forceinline__ void stage_weight(const TIn* __restrict__ W, float* __restrict__ rm) {
  constexpr int kLd = D + 4;
  constexpr int kPer = 16 / (int)sizeof(TIn);  // elements per 16-byte load
  for (int i = threadIdx.x; i < D * D / kPer; i += blockDim.x) {
    const int row = (i * kPer) / D, col0 = (i * kPer) % D;  // W[row][col0 .. col0 + kPer)
    float f[kPer];
    if constexpr (sizeof(TIn) == 2) {
      const uint4 raw = reinterpret_cast<const uint4*>(W)[i];
      const uint32_t w32[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f[2 * q] = __uint_as_float(w32[q] << 16);
        f[2 * q + 1] = __uint_as_float(w32[q] & 0xFFFF0000u);
      }
    } else {
      const float4 v = reinterpret_cast<const float4*>(W)[i];
      f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    if constexpr (kTranspose) {
#pragma unroll
      for (int q = 0; q < kPer; ++q) rm[(col0 + q) * kLd + row] = f[q];
    } else {
#pragma unroll
      for (int q = 0; q < kPer; q += 4)
        *reinterpret_cast<float4*>(rm + row * kLd + col0 + q) = make_float4(f[q], f[q + 1], f[q + 2], f[q + 3]);
    }
  }
}

template <int D, int RT = kRowTile>
__device__ __forceinline__ void tile_gemm(const float* __restrict__ lr, const float* __restrict__ rm,
                                          float (&acc)[TileShape<D, RT>::kJPT][4]) {
  using S = TileShape<D, RT>;
  const int te = threadIdx.x % S::kTE, tj = threadIdx.x / S::kTE;
#pragma unroll
  for (int r = 0; r < S::kJPT; ++r)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[r][x] = 0.f;
#pragma unroll 2
  for (int c = 0; c < D; c += 4) {
    float4 w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = *reinterpret_cast<const float4*>(rm + (c + q) * S::kLd + te * 4);
#pragma unroll
    for (int r = 0; r < S::kJPT; ++r) {
      const float4 l = *reinterpret_cast<const float4*>(lr + (tj * S::kJPT + r) * S::kLd + c);
      const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[r][0] = fmaf(lv[q], w[q].x, acc[r][0]);
        acc[r][1] = fmaf(lv[q], w[q].y, acc[r][1]);
        acc[r][2] = fmaf(lv[q], w[q].z, acc[r][2]);
        acc[r][3] = fmaf(lv[q], w[q].w, acc[r][3]);
      }
    }
  }
}

// fold, tiled: block = 16 prototypes; Pf[j][c] = scale * sum_e P[j][e] Wk[c][e].
template <int D, typename TIn>
__global__ void __launch_bounds__(256) fold_tiled_kernel(const TIn* __restrict__ P,
                                                         const TIn* __restrict__ Wk, int k,
                                                         int k_pad, float scale,
                                                         void* __restrict__ out, int out_bf16) {
  using S = TileShape<D, kFoldRowTile>;
  extern __shared__ __align__(16) float tsm[];
  float* lr = tsm;                          // [16][D+4]  lr[j][e] = P[j0 + j][e]
  float* rm = tsm + kFoldRowTile * S::kLd;  // [D][D+4]   rm[e][c] = Wk[c][e]
  const int j0 = blockIdx.x * kFoldRowTile;
  for (int i = threadIdx.x; i < kFoldRowTile * D; i += blockDim.x) {
    const int j = i / D, e = i % D;
    lr[j * S::kLd + e] = (j0 + j < k) ? to_f(P[(size_t)(j0 + j) * D + e]) : 0.f;
  }
  stage_weight<D, TIn, true>(Wk, rm);
  __syncthreads();
  float acc[S::kJPT][4];
  tile_gemm<D, kFoldRowTile>(lr, rm, acc);
  const int te = threadIdx.x % S::kTE, tj = threadIdx.x / S::kTE;
#pragma unroll
  for (int r = 0; r < S::kJPT; ++r) {
    const int j = j0 + tj * S::kJPT + r;
    if (j >= k_pad) continue;
    const size_t o = (size_t)j * D + te * 4;
    if (out_bf16) {
      __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(out) + o;
      ob[0] = __float2bfloat16_rn(acc[r][0] * scale);
      ob[1] = __float2bfloat16_rn(acc[r][1] * scale);
      ob[2] = __float2bfloat16_rn(acc[r][2] * scale);
      ob[3] = __float2bfloat16_rn(acc[r][3] * scale);
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o) =
          make_float4(acc[r][0] * scale, acc[r][1] * scale, acc[r][2] * scale, acc[r][3] * scale);
    }
  }
}

// finalize, tiled: block = (user u, 64 prototypes). Adds the user's segment partials in
// range order (deterministic), writes xsketch = U and mass, then sketch = U Wv / mass.
template <int D, typename TIn>
__global__ void __launch_bounds__(256) finalize_tiled_kernel(FinalizeArgs a, const TIn* __restrict__ Wv) {
  using S = TileShape<D>;
  extern __shared__ __align__(16) float tsm[];
  float* lr = tsm;                      // [64][D+4]  lr[j][c] = U[j0 + j][c]
  float* rm = tsm + kRowTile * S::kLd;  // [D][D+4]   rm[c][e] = Wv[c][e]
  float* ms = rm + D * S::kLd;          // [64]
  constexpr int kV = D / 4;             // float4 per row
  const int u = blockIdx.x;
  const int j0 = blockIdx.y * kRowTile;
  if (read_status(&a.hdr->status) != 0) return;
  const long long T = a.hdr->total_tiles;
  const long long x0 = a.tile_start[u], x1 = a.tile_start[u + 1];
  float4 us[kRowTile * kV / 256];       // this thread's float4 of the U tile
  float mv = 0.f;                       // thread t < 64: mass of row t
#pragma unroll
  for (int q = 0; q < kRowTile * kV / 256; ++q) us[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (x1 > x0) {
    const TileRanges rg(T, a.G, a.H, a.share);
    const int g0 = rg.of_tile(x0), g1 = rg.of_tile(x1 - 1);
    for (int g = g0; g <= g1; ++g) {
      if (rg.start(g) == rg.start(g + 1)) continue;  // empty range
      const size_t seg = (size_t)g + u;
      const float4* src = reinterpret_cast<const float4*>(a.part_u + (seg * a.k_pad + j0) * D);
#pragma unroll
      for (int q = 0; q < kRowTile * kV / 256; ++q) {
        const int i = threadIdx.x + q * 256;
        if (j0 + i / kV < a.k_pad) {
          const float4 v = src[i];
          us[q].x += v.x; us[q].y += v.y; us[q].z += v.z; us[q].w += v.w;
        }
      }
      if (threadIdx.x < kRowTile && j0 + (int)threadIdx.x < a.k_pad) {
        const float* pm = a.part_m + (seg * a.k_pad + j0 + threadIdx.x) * a.mass_lanes;
        float v = 0.f;
        for (int l = 0; l < a.mass_lanes; ++l) v += pm[l];
        mv += v;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kRowTile * kV / 256; ++q) {
    const int i = threadIdx.x + q * 256;
    const int j = i / kV, c4 = i % kV;
    *reinterpret_cast<float4*>(lr + j * S::kLd + c4 * 4) = us[q];
    if (a.xsketch && j0 + j < a.k)
      reinterpret_cast<float4*>(a.xsketch + ((size_t)u * a.k + j0 + j) * D)[c4] = us[q];
  }
  if (threadIdx.x < kRowTile) {
    ms[threadIdx.x] = mv;
    if (j0 + (int)threadIdx.x < a.k) a.mass[(size_t)u * a.k + j0 + threadIdx.x] = mv;
  }
  stage_weight<D, TIn, false>(Wv, rm);
  __syncthreads();
  float acc[S::kJPT][4];
  tile_gemm<D>(lr, rm, acc);
  const int te = threadIdx.x % S::kTE, tj = threadIdx.x / S::kTE;
#pragma unroll
  for (int r = 0; r < S::kJPT; ++r) {
    const int jj = tj * S::kJPT + r, j = j0 + jj;
    if (j >= a.k) continue;
    const float m = ms[jj];
    const float inv = m > 0.f ? 1.f / m : 0.f;
    *reinterpret_cast<float4*>(a.sketch + ((size_t)u * a.k + j) * D + te * 4) =
        make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
  }
}

// finalize, split: block = (user u, 64 prototypes). Adds the user's segment partials in
// range order (deterministic), writes xsketch = U and mass, and U / mass (0 where
// mass = 0) as a bf16 pair hi + lo with hi + lo = U / mass to about 16 bits; the product
// with Wv runs on the tensor cores as two accumulated GEMM phases (hi Wv + lo Wv).
template <int D>
__global__ void __launch_bounds__(256) finalize_split_kernel(FinalizeArgs a) {
  constexpr int kV = D / 4;                 // float4 per row
  constexpr int kQ = kRowTile * kV / 256;   // float4 of the U tile per thread
  __shared__ float ms[kRowTile];
  const int u = blockIdx.x;
  const int j0 = blockIdx.y * kRowTile;
  if (read_status(&a.hdr->status) != 0) return;
  const long long T = a.hdr->total_tiles;
  const long long x0 = a.tile_start[u], x1 = a.tile_start[u + 1];
  float4 us[kQ];
  float mv = 0.f;
#pragma unroll
  for (int q = 0; q < kQ; ++q) us[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (x1 > x0) {
    const TileRanges rg(T, a.G, a.H, a.share);
    const int g0 = rg.of_tile(x0), g1 = rg.of_tile(x1 - 1);
    for (int g = g0; g <= g1; ++g) {
      if (rg.start(g) == rg.start(g + 1)) continue;  // empty range
      const size_t seg = (size_t)g + u;
      const float4* src = reinterpret_cast<const float4*>(a.part_u + (seg * a.k_pad + j0) * D);
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const float4 v = src[threadIdx.x + q * 256];
        us[q].x += v.x; us[q].y += v.y; us[q].z += v.z; us[q].w += v.w;
      }
      if (threadIdx.x < kRowTile) {
        const float* pm = a.part_m + (seg * a.k_pad + j0 + threadIdx.x) * a.mass_lanes;
        float v = 0.f;
        for (int l = 0; l < a.mass_lanes; ++l) v += pm[l];
        mv += v;
      }
    }
  }
  if (threadIdx.x < kRowTile) {
    ms[threadIdx.x] = mv;
    a.mass[(size_t)u * a.k + j0 + threadIdx.x] = mv;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    const int i = threadIdx.x + q * 256;
    const int j = i / kV, c4 = i % kV;
    const size_t row = (size_t)u * a.k + j0 + j;
    if (a.xsketch) reinterpret_cast<float4*>(a.xsketch + row * D)[c4] = us[q];
    const float m = ms[j];
    const float inv = m > 0.f ? 1.f / m : 0.f;
    const float v[4] = {us[q].x * inv, us[q].y * inv, us[q].z * inv, us[q].w * inv};
    uint32_t hi[2], lo[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * h]), h1 = __float2bfloat16_rn(v[2 * h + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * h] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * h + 1] - __bfloat162float(h1));
      hi[h] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[h] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    reinterpret_cast<uint2*>(a.ubar_hi + row * D)[c4] = make_uint2(hi[0], hi[1]);
    reinterpret_cast<uint2*>(a.ubar_lo + row * D)[c4] = make_uint2(lo[0], lo[1]);
  }
}

// combine, tiled: block = (user u, 64 prototypes). U and mass are already summed (over
// the parts of a user that was split across calls); sketch = U Wv / mass.
template <int D, typename TIn>
__global__ void __launch_bounds__(256) combine_tiled_kernel(const float* __restrict__ U,
                                                            const float* __restrict__ mass, int k,
                                                            const TIn* __restrict__ Wv,
                                                            float* __restrict__ sketch) {
  using S = TileShape<D>;
  extern __shared__ __align__(16) float tsm[];
  float* lr = tsm;                      // [64][D+4]
  float* rm = tsm + kRowTile * S::kLd;  // [D][D+4]
  float* ms = rm + D * S::kLd;          // [64]
  constexpr int kV = D / 4;
  const int u = blockIdx.x;
  const int j0 = blockIdx.y * kRowTile;
  for (int i = threadIdx.x; i < kRowTile * kV; i += blockDim.x) {
    const int j = i / kV, c4 = i % kV;
    const float4 v = (j0 + j < k)
        ? reinterpret_cast<const float4*>(U + ((size_t)u * k + j0 + j) * D)[c4]
        : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(lr + j * S::kLd + c4 * 4) = v;
  }
  if (threadIdx.x < kRowTile)
    ms[threadIdx.x] = (j0 + (int)threadIdx.x < k) ? mass[(size_t)u * k + j0 + threadIdx.x] : 0.f;
  stage_weight<D, TIn, false>(Wv, rm);
  __syncthreads();
  float acc[S::kJPT][4];
  tile_gemm<D>(lr, rm, acc);
  const int te = threadIdx.x % S::kTE, tj = threadIdx.x / S::kTE;
#pragma unroll
  for (int r = 0; r < S::kJPT; ++r) {
    const int jj = tj * S::kJPT + r, j = j0 + jj;
    if (j >= k) continue;
    const float m = ms[jj];
    const float inv = m > 0.f ? 1.f / m : 0.f;
    *reinterpret_cast<float4*>(sketch + ((size_t)u * k + j) * D + te * 4) =
        make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
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

template <int D, typename TIn>
cudaError_t launch_fold_t(const void* P, const void* Wk, int k, int k_pad, float scale, void* Pf,
                          bool out_bf16, cudaStream_t s) {
  auto kern = fold_tiled_kernel<D, TIn>;
  const size_t smem = (size_t)(kFoldRowTile + D) * TileShape<D, kFoldRowTile>::kLd * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((k_pad + kFoldRowTile - 1) / kFoldRowTile));
  kern<<<grid, 256, smem, s>>>(static_cast<const TIn*>(P), static_cast<const TIn*>(Wk), k, k_pad,
                               scale, Pf, out_bf16 ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_fold(const void* P, const void* Wk, sa_dtype dt, int k, int k_pad, int d,
                        float scale, void* Pf, bool out_bf16, cudaStream_t s) {
  if (dt == SA_BF16)
    return d == 128 ? launch_fold_t<128, __nv_bfloat16>(P, Wk, k, k_pad, scale, Pf, out_bf16, s)
                    : launch_fold_t<64, __nv_bfloat16>(P, Wk, k, k_pad, scale, Pf, out_bf16, s);
  return d == 128 ? launch_fold_t<128, float>(P, Wk, k, k_pad, scale, Pf, out_bf16, s)
                  : launch_fold_t<64, float>(P, Wk, k, k_pad, scale, Pf, out_bf16, s);
}

template <int D, typename TIn>
cudaError_t launch_finalize_t(const FinalizeArgs& a, cudaStream_t s) {
  auto kern = finalize_tiled_kernel<D, TIn>;
  const size_t smem = ((size_t)(kRowTile + D) * TileShape<D>::kLd + kRowTile) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)a.R, (unsigned)((a.k + kRowTile - 1) / kRowTile));
  kern<<<grid, 256, smem, s>>>(a, static_cast<const TIn*>(a.Wv));
  return cudaGetLastError();
}

cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t s) {
  if (a.R == 0) return cudaSuccess;
  if (a.dt == SA_BF16)
    return a.d == 128 ? launch_finalize_t<128, __nv_bfloat16>(a, s) : launch_finalize_t<64, __nv_bfloat16>(a, s);
  return a.d == 128 ? launch_finalize_t<128, float>(a, s) : launch_finalize_t<64, float>(a, s);
}

cudaError_t launch_finalize_tc(const FinalizeArgs& a, cudaStream_t s) {
  if (a.R == 0) return cudaSuccess;
  if (a.dt != SA_BF16 || a.k != a.k_pad || !a.ubar_hi || !a.ubar_lo) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)a.R, (unsigned)(a.k / kRowTile));
  if (a.d == 128)
    finalize_split_kernel<128><<<grid, 256, 0, s>>>(a);
  else
    finalize_split_kernel<64><<<grid, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  GemmArgs g = {};
  const uint64_t rows = (uint64_t)a.R * a.k;
  g.a[0] = {a.ubar_hi, rows, (uint64_t)a.d, false};
  g.a[1] = {a.ubar_lo, rows, (uint64_t)a.d, false};
  g.b[0] = {a.Wv, (uint64_t)a.d, (uint64_t)a.d, true};  // Wv[c][e]: rows = K, cols = N
  g.b[1] = g.b[0];
  g.phases = 2;
  g.k_tiles[0] = g.k_tiles[1] = a.d / 64;
  g.M = (int)rows;
  g.N = a.d;
  g.m_tiles_bound = (int)((rows + 127) / 128);
  g.splits = 1;
  g.epi = kEpiStoreF32;
  g.hdr = a.hdr;
  g.out_f32 = a.sketch;
  g.ld_out = a.d;
  return launch_gemm(g, s);
}

template <int D, typename TIn>
cudaError_t launch_combine_t(const float* U, const float* mass, int R, int k, const void* Wv,
                             float* sketch, cudaStream_t s) {
  auto kern = combine_tiled_kernel<D, TIn>;
  const size_t smem = ((size_t)(kRowTile + D) * TileShape<D>::kLd + kRowTile) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)R, (unsigned)((k + kRowTile - 1) / kRowTile));
  kern<<<grid, 256, smem, s>>>(U, mass, k, static_cast<const TIn*>(Wv), sketch);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* U, const float* mass, int R, int k, int d, const void* Wv,
                           sa_dtype dt, float* sketch, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  if (dt == SA_BF16)
    return d == 128 ? launch_combine_t<128, __nv_bfloat16>(U, mass, R, k, Wv, sketch, s)
                    : launch_combine_t<64, __nv_bfloat16>(U, mass, R, k, Wv, sketch, s);
  return d == 128 ? launch_combine_t<128, float>(U, mass, R, k, Wv, sketch, s)
                  : launch_combine_t<64, float>(U, mass, R, k, Wv, sketch, s);
}

cudaError_t launch_debug_wait_timeout(WsHeader* hdr, long long budget, cudaStream_t s) {
  debug_wait_timeout_kernel<<<1, 32, 0, s>>>(hdr, budget);
  return cudaGetLastError();
}

}  // namespace sa
