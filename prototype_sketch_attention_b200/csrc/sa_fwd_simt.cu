// Sketch Attention forward for fp32 inputs on CUDA cores (tcgen05 has no fp32-input
// MMA, and tf32 would not hold the fp32 path's 1e-5 tolerance).
//
// Same definition as the tensor-core path (blog "100,000 videos in your pocket",
// section "1. Sketch Attention compresses the history"): with the folded prototypes
// Pf = P W_k^T log2(e)/sqrt(d) the log2-unit score is s_jt = Pf_j . X_t.
//   kernel 1: per token, lse2_t = log2 sum_j 2^(s_jt)  (online over prototype chunks)
//   kernel 2: per (token-range worker, 32 prototypes): A_jt = 2^(s_jt - lse2_t),
//             U_j += A_jt X_t, mass_j += A_jt; a partial per (worker, user) segment,
//             summed later in worker order by the finalize kernel.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kLseTok = 64;    // tokens per block in kernel 1
constexpr int kChunkP = 32;    // prototypes per chunk

__global__ void __launch_bounds__(256) lse_simt_kernel(const float* __restrict__ X, int64_t n_total,
                                                       int d, const float* __restrict__ Pf, int k,
                                                       const WsHeader* __restrict__ hdr,
                                                       float* __restrict__ lse2,
                                                       float* __restrict__ lse) {
  extern __shared__ float sm[];
  const int ld = d + 1;
  float* xs = sm;                  // [64][d+1]
  float* ps = sm + kLseTok * ld;   // [32][d+1]
  if (read_status(&hdr->status) != 0) return;
  const int64_t t0 = (int64_t)blockIdx.x * kLseTok;
  for (int i = threadIdx.x; i < kLseTok * d; i += blockDim.x) {
    const int r = i / d, c = i % d;
    xs[r * ld + c] = (t0 + r < n_total) ? X[(t0 + r) * d + c] : 0.f;
  }
  const int tok = threadIdx.x >> 2;      // 0..63
  const int p0 = (threadIdx.x & 3) * 8;  // 8 prototypes per thread per chunk
  float m = -INFINITY, z = 0.f;
  for (int j0 = 0; j0 < k; j0 += kChunkP) {
    __syncthreads();
    for (int i = threadIdx.x; i < kChunkP * d; i += blockDim.x) {
      const int r = i / d, c = i % d;
      ps[r * ld + c] = Pf[(size_t)(j0 + r) * d + c];
    }
    __syncthreads();
    float s[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) s[p] = 0.f;
    for (int c = 0; c < d; ++c) {
      const float x = xs[tok * ld + c];
#pragma unroll
      for (int p = 0; p < 8; ++p) s[p] = fmaf(x, ps[(p0 + p) * ld + c], s[p]);
    }
    float cm = -INFINITY;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      if (j0 + p0 + p >= k) s[p] = -INFINITY;
      cm = fmaxf(cm, s[p]);
    }
    cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
    cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
    float cz = 0.f;
#pragma unroll
    for (int p = 0; p < 8; ++p) cz += exp2f(s[p] - cm);
    cz += __shfl_xor_sync(0xffffffffu, cz, 1);
    cz += __shfl_xor_sync(0xffffffffu, cz, 2);
    const float nm = fmaxf(m, cm);
    z = z * exp2f(m - nm) + cz * exp2f(cm - nm);
    m = nm;
  }
  if ((threadIdx.x & 3) == 0 && t0 + tok < n_total) {
    const float l2 = m + log2f(z);
    lse2[t0 + tok] = l2;
    if (lse) lse[t0 + tok] = l2 * 0.69314718055994530942f;
  }
}

// Block (worker g, prototypes [32 by, 32 by + 32)); walks tiles [a_g, b_g).
__global__ void __launch_bounds__(256) accum_simt_kernel(FwdSimtArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, ld = d + 1;
  float* xs = sm;                        // [128][d+1]
  float* ps = xs + kTileTokens * ld;     // [32][d+1]
  float* as = ps + kChunkP * ld;         // [32][129]
  float* ls = as + kChunkP * 129;        // [128]
  if (read_status(&a.hdr->status) != 0) return;
  const long long T = a.hdr->total_tiles;
  const int g = blockIdx.x, G = gridDim.x;
  const long long ta = (long long)g * T / G, tb = (long long)(g + 1) * T / G;
  const int j0 = blockIdx.y * kChunkP;
  for (int i = threadIdx.x; i < kChunkP * d; i += blockDim.x) {
    const int r = i / d, c = i % d;
    ps[r * ld + c] = a.Pf[(size_t)(j0 + r) * d + c];
  }
  // accumulator ownership: e = t % d, prototypes jg + js*i
  const int e = threadIdx.x % d, jg = threadIdx.x / d, js = blockDim.x / d;
  const int nacc = kChunkP / js;  // 16 (d=128) or 8 (d=64)
  float acc[16];
  float macc = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  TileIter it;
  it.init(a.tile_start, a.offsets, a.R, ta, tb);
  for (; it.valid(); it.next()) {
    const long long t0 = it.t0();
    const int nv = it.nvalid();
    __syncthreads();
    for (int i = threadIdx.x; i < kTileTokens * d; i += blockDim.x) {
      const int r = i / d, c = i % d;
      xs[r * ld + c] = (r < nv) ? a.X[(t0 + r) * d + c] : 0.f;
    }
    if (threadIdx.x < kTileTokens) ls[threadIdx.x] = threadIdx.x < nv ? a.lse2[t0 + threadIdx.x] : 0.f;
    __syncthreads();
    {
      // A[j][tok] for 32 x 128 pairs: thread -> prototype j = t / 8, tokens 16 (t % 8) .. +16
      const int j = threadIdx.x >> 3, tb0 = (threadIdx.x & 7) * 16;
      float s[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) s[q] = 0.f;
      for (int c = 0; c < d; ++c) {
        const float pv = ps[j * ld + c];
#pragma unroll
        for (int q = 0; q < 16; ++q) s[q] = fmaf(pv, xs[(tb0 + q) * ld + c], s[q]);
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int tok = tb0 + q;
        as[j * 129 + tok] = (tok < nv && j0 + j < a.k) ? exp2f(s[q] - ls[tok]) : 0.f;
      }
    }
    __syncthreads();
    for (int i = 0; i < nacc; ++i) {
      const int j = jg + js * i;
      float v = 0.f;
      for (int tok = 0; tok < nv; ++tok) v = fmaf(as[j * 129 + tok], xs[tok * ld + e], v);
      acc[i] += v;
    }
    if (threadIdx.x < kChunkP) {
      float v = 0.f;
      for (int tok = 0; tok < nv; ++tok) v += as[threadIdx.x * 129 + tok];
      macc += v;
    }
    if (it.last()) {
      const size_t seg = (size_t)g + it.u;
      for (int i = 0; i < nacc; ++i) {
        const int j = jg + js * i;
        a.part_u[(seg * a.k_pad + j0 + j) * d + e] = acc[i];
        acc[i] = 0.f;
      }
      if (threadIdx.x < kChunkP) {
        a.part_m[seg * a.k_pad + j0 + threadIdx.x] = macc;
        macc = 0.f;
      }
    }
  }
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdSimtArgs& a, cudaStream_t s) {
  if (a.n_total > 0) {
    const size_t smem1 = (size_t)(kLseTok + kChunkP) * (a.d + 1) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(lse_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    const unsigned nb = (unsigned)((a.n_total + kLseTok - 1) / kLseTok);
    lse_simt_kernel<<<nb, 256, smem1, s>>>(a.X, a.n_total, a.d, a.Pf, a.k, a.hdr, a.lse2, a.lse);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem2 =
        (size_t)((kTileTokens + kChunkP) * (a.d + 1) + kChunkP * 129 + kTileTokens) * sizeof(float);
    e = cudaFuncSetAttribute(accum_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    if (e != cudaSuccess) return e;
    accum_simt_kernel<<<dim3((unsigned)a.G, (unsigned)(a.k_pad / kChunkP)), 256, smem2, s>>>(a);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace sa
