// Sketch Attention backward on CUDA cores (fp32 arithmetic; bf16 or fp32 inputs).
//
// Sketch Attention is differentiable: the ranking loss's gradient flows back through
// the compression (blog "100,000 videos in your pocket", section "1. Sketch Attention
// compresses the history"). With Pn = P W_k^T / sqrt(d) (so s_jt = Pn_j . X_t),
// G = dL/dsketch, Gm = dL/dmass, and per user:
//   Gt_j = G_j / mass_j,  Gh_j = Gt_j W_v^T,  c_j = Gt_j . sketch_j - Gm_j
//   dA_jt = Gh_j . X_t - c_j,   D_t = sum_j A_jt dA_jt,   dS_jt = A_jt (dA_jt - D_t)
//   dX_t  = sum_j dS_jt Pn_j + sum_j A_jt Gh_j
//   dPn   = sum_users sum_t dS_jt X_t
//   dP    = dPn W_k / sqrt(d),  dW_k = dPn^T P / sqrt(d),  dW_v = sum_users U^T Gt
// where U = sum_t A_jt X_t is the forward's xsketch. The per-token statistics
// (lse_t, D_t) are recomputed here in fp32 from the unrounded Pn.
// Every reduction over tokens or users is split into fixed chunks added in a fixed
// order, so the result is deterministic.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kCP = 32;   // prototypes per chunk
constexpr int kWvRows = 1024;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float* p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

// ---- per-user prep: Gt, c, and Gh unless a GEMM computes it (Gtlo given: then Gt's bf16
// hi and lo parts).   grid (R, k_pad/32), 256 threads
template <typename TIn>
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdArgs a, const TIn* __restrict__ Wv) {
  extern __shared__ float sm[];
  const int d = a.d, ld = d + 1;
  float* gt = sm;              // [32][d]
  float* wv = sm + kCP * d;    // [d][d+1]  wv[c][e] = Wv[c][e] (only without Gtlo)
  const int u = blockIdx.x, j0 = blockIdx.y * kCP;
  if (!a.Gtlo)  // W_v is needed here only when this kernel computes Gh itself
    for (int i = threadIdx.x; i < d * d; i += blockDim.x) wv[(i / d) * ld + (i % d)] = ldf(Wv, i);
  for (int i = threadIdx.x; i < kCP * d; i += blockDim.x) {
    const int jj = i / d, e = i % d, j = j0 + jj;
    float v = 0.f;
    if (j < a.k) {
      const float m = a.mass[(size_t)u * a.k + j];
      v = m > 0.f ? a.dsketch[((size_t)u * a.k + j) * d + e] / m : 0.f;
    }
    gt[i] = v;
    a.Gt[((size_t)u * a.k_pad + j) * d + e] = v;
    if (a.Gtb) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      a.Gtb[((size_t)u * a.k_pad + j) * d + e] = hi;
      if (a.Gtlo) a.Gtlo[((size_t)u * a.k_pad + j) * d + e] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < (a.Gtlo ? 0 : kCP * d); i += blockDim.x) {  // else a GEMM
    const int jj = i / d, c = i % d;
    float acc = 0.f;
    for (int e = 0; e < d; ++e) acc = fmaf(gt[jj * d + e], wv[c * ld + e], acc);
    const size_t o = ((size_t)u * a.k_pad + j0 + jj) * d + c;
    if (a.Gh) a.Gh[o] = acc;
    if (a.Ghb) a.Ghb[o] = __float2bfloat16_rn(acc);
  }
  // c_j = Gt_j . sketch_j - dmass_j: each warp takes kCP / 8 rows, its lanes read the
  // sketch row coalesced, and a shuffle tree adds the lanes
  for (int jj = threadIdx.x >> 5; jj < kCP; jj += blockDim.x >> 5) {
    const int j = j0 + jj, lane = threadIdx.x & 31;
    float v = 0.f;
    if (j < a.k)
      for (int e = lane; e < d; e += 32)
        v = fmaf(gt[jj * d + e], a.sketch[((size_t)u * a.k + j) * d + e], v);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      if (j < a.k && a.dmass) v -= a.dmass[(size_t)u * a.k + j];
      a.cj[(size_t)u * a.k_pad + j] = j < a.k ? v : 0.f;
    }
  }
}

// ---- token owner: dX, lse_t, D_t.   grid = total tiles, 256 threads, 128 tokens
template <typename TIn>
__global__ void __launch_bounds__(256) bwd_token_kernel(BwdArgs a, const TIn* __restrict__ X) {
  extern __shared__ float sm[];
  const int d = a.d, ld = d + 1;
  float* xs = sm;                     // [128][d+1]
  float* ps = xs + kTileTokens * ld;  // [32][d+1]
  float* gs = ps + kCP * ld;          // [32][d+1]
  float* as = gs + kCP * ld;          // [128][33]
  float* ds = as + kTileTokens * 33;  // [128][33]
  float* cs = ds + kTileTokens * 33;  // [32]
  if (read_status(&a.hdr->status) != 0) return;
  const long long tile = blockIdx.x;
  if (tile >= a.hdr->total_tiles) return;
  const int u = user_of_tile(a.tile_start, a.R, tile);
  const long long local = tile - a.tile_start[u];
  const long long t0 = a.offsets[u] + local * kTileTokens;
  const long long nrem = a.offsets[u + 1] - t0;
  const int nv = nrem >= kTileTokens ? kTileTokens : (int)nrem;
  for (int i = threadIdx.x; i < kTileTokens * d; i += blockDim.x) {
    const int r = i / d, c = i % d;
    xs[r * ld + c] = r < nv ? ldf(X, (size_t)(t0 + r) * d + c) : 0.f;
  }
  const int tok = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int p0 = half * 16;
  const float* Gh_u = a.Gh + (size_t)u * a.k_pad * d;
  const float* c_u = a.cj + (size_t)u * a.k_pad;

  auto load_chunk = [&](int j0) {
    __syncthreads();
    for (int i = threadIdx.x; i < kCP * d; i += blockDim.x) {
      const int r = i / d, c = i % d;
      ps[r * ld + c] = a.Pn[(size_t)(j0 + r) * d + c];
      gs[r * ld + c] = Gh_u[(size_t)(j0 + r) * d + c];
    }
    if (threadIdx.x < kCP) cs[threadIdx.x] = c_u[j0 + threadIdx.x];
    __syncthreads();
  };
  auto scores = [&](float (&s)[16], float (&g)[16]) {
#pragma unroll
    for (int p = 0; p < 16; ++p) { s[p] = 0.f; g[p] = 0.f; }
    for (int c = 0; c < d; ++c) {
      const float x = xs[tok * ld + c];
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        s[p] = fmaf(x, ps[(p0 + p) * ld + c], s[p]);
        g[p] = fmaf(x, gs[(p0 + p) * ld + c], g[p]);
      }
    }
  };

  // pass 1: online (max, sum e, sum e dA) over prototypes
  float m = -INFINITY, z = 0.f, w = 0.f;
  for (int j0 = 0; j0 < a.k; j0 += kCP) {
    load_chunk(j0);
    float s[16], g[16];
    scores(s, g);
    float cm = -INFINITY;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      if (j0 + p0 + p >= a.k) s[p] = -INFINITY;
      cm = fmaxf(cm, s[p]);
    }
    const float nm = fmaxf(m, cm);
    float cz = 0.f, cw = 0.f;
    if (nm > -INFINITY) {
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const float ev = __expf(s[p] - nm);
        cz += ev;
        cw = fmaf(ev, g[p] - cs[p0 + p], cw);
      }
      const float r = (m > -INFINITY) ? __expf(m - nm) : 0.f;
      z = z * r + cz;
      w = w * r + cw;
      m = nm;
    }
  }
  {
    const float om = __shfl_xor_sync(0xffffffffu, m, 1);
    const float oz = __shfl_xor_sync(0xffffffffu, z, 1);
    const float ow = __shfl_xor_sync(0xffffffffu, w, 1);
    const float nm = fmaxf(m, om);
    const float r0 = (m > -INFINITY) ? __expf(m - nm) : 0.f;
    const float r1 = (om > -INFINITY) ? __expf(om - nm) : 0.f;
    z = z * r0 + oz * r1;
    w = w * r0 + ow * r1;
    m = nm;
  }
  const float lse = m + __logf(z);
  const float D = w / z;
  if (half == 0 && tok < nv) {
    a.lseb[t0 + tok] = lse;
    a.Db[t0 + tok] = D;
  }

  // pass 2: dS, A -> dX
  float acc[64];
  const int e0 = half * (d / 2);
  const int ne = d / 2;
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = 0.f;
  for (int j0 = 0; j0 < a.k; j0 += kCP) {
    load_chunk(j0);
    float s[16], g[16];
    scores(s, g);
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const bool ok = (j0 + p0 + p < a.k) && tok < nv;
      const float A = ok ? __expf(s[p] - lse) : 0.f;
      as[tok * 33 + p0 + p] = A;
      ds[tok * 33 + p0 + p] = A * (g[p] - cs[p0 + p] - D);
    }
    __syncthreads();
    for (int p = 0; p < kCP; ++p) {
      const float av = as[tok * 33 + p], dv = ds[tok * 33 + p];
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (i < ne) acc[i] = fmaf(dv, ps[p * ld + e0 + i], fmaf(av, gs[p * ld + e0 + i], acc[i]));
    }
  }
  if (tok < nv) {
#pragma unroll
    for (int i = 0; i < 64; ++i)
      if (i < ne) a.dX[(size_t)(t0 + tok) * d + e0 + i] = acc[i];
  }
}

// ---- prototype owner: dPn partials per worker.   grid (G, k_pad/32), 256 threads
template <typename TIn>
__global__ void __launch_bounds__(256) bwd_proto_kernel(BwdArgs a, const TIn* __restrict__ X) {
  extern __shared__ float sm[];
  const int d = a.d, ld = d + 1;
  float* xs = sm;                     // [128][d+1]
  float* ps = xs + kTileTokens * ld;  // [32][d+1]
  float* gs = ps + kCP * ld;          // [32][d+1]
  float* dss = gs + kCP * ld;         // [32][129]
  float* ls = dss + kCP * 129;        // [128] lse
  float* Ds = ls + kTileTokens;       // [128] D
  float* cs = Ds + kTileTokens;       // [32]
  if (read_status(&a.hdr->status) != 0) return;
  const long long T = a.hdr->total_tiles;
  const int gw = blockIdx.x, G = gridDim.x;
  const long long ta = (long long)gw * T / G, tb = (long long)(gw + 1) * T / G;
  const int j0 = blockIdx.y * kCP;
  for (int i = threadIdx.x; i < kCP * d; i += blockDim.x) {
    const int r = i / d, c = i % d;
    ps[r * ld + c] = a.Pn[(size_t)(j0 + r) * d + c];
  }
  const int e = threadIdx.x % d, jg = threadIdx.x / d, js = blockDim.x / d;
  const int nacc = kCP / js;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  TileIter it;
  it.init(a.tile_start, a.offsets, a.R, ta, tb);
  int cur_u = -1;
  for (; it.valid(); it.next()) {
    const long long t0 = it.t0();
    const int nv = it.nvalid();
    __syncthreads();
    if (it.u != cur_u) {
      cur_u = it.u;
      const float* Gh_u = a.Gh + (size_t)cur_u * a.k_pad * d;
      for (int i = threadIdx.x; i < kCP * d; i += blockDim.x) {
        const int r = i / d, c = i % d;
        gs[r * ld + c] = Gh_u[(size_t)(j0 + r) * d + c];
      }
      if (threadIdx.x < kCP) cs[threadIdx.x] = a.cj[(size_t)cur_u * a.k_pad + j0 + threadIdx.x];
    }
    for (int i = threadIdx.x; i < kTileTokens * d; i += blockDim.x) {
      const int r = i / d, c = i % d;
      xs[r * ld + c] = r < nv ? ldf(X, (size_t)(t0 + r) * d + c) : 0.f;
    }
    if (threadIdx.x < kTileTokens) {
      const bool v = threadIdx.x < nv;
      ls[threadIdx.x] = v ? a.lseb[t0 + threadIdx.x] : 0.f;
      Ds[threadIdx.x] = v ? a.Db[t0 + threadIdx.x] : 0.f;
    }
    __syncthreads();
    {
      const int j = threadIdx.x >> 3, tb0 = (threadIdx.x & 7) * 16;
      float s[16], g[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) { s[q] = 0.f; g[q] = 0.f; }
      for (int c = 0; c < d; ++c) {
        const float pv = ps[j * ld + c], gv = gs[j * ld + c];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float x = xs[(tb0 + q) * ld + c];
          s[q] = fmaf(pv, x, s[q]);
          g[q] = fmaf(gv, x, g[q]);
        }
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int tok = tb0 + q;
        float v = 0.f;
        if (tok < nv && j0 + j < a.k) {
          const float A = __expf(s[q] - ls[tok]);
          v = A * (g[q] - cs[j] - Ds[tok]);
        }
        dss[j * 129 + tok] = v;
      }
    }
    __syncthreads();
    for (int i = 0; i < nacc; ++i) {
      const int j = jg + js * i;
      float v = 0.f;
      for (int tok = 0; tok < nv; ++tok) v = fmaf(dss[j * 129 + tok], xs[tok * ld + e], v);
      acc[i] += v;
    }
  }
  for (int i = 0; i < nacc; ++i) {
    const int j = jg + js * i;
    a.dpp_part[((size_t)gw * a.k_pad + j0 + j) * d + e] = acc[i];
  }
}

// ---- dPn = sum over workers (fixed order)
__global__ void bwd_reduce_dpp_kernel(BwdArgs a) {
  if (read_status(&a.hdr->status) != 0) return;
  const size_t n = (size_t)a.k_pad * a.d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int g = 0; g < a.G; ++g) v += a.dpp_part[(size_t)g * n + i];
    a.dpp[i] = v;
  }
}

// ---- dW_v partials: rows r = (u, j) in chunks of 1024.   grid = nchunks, 256 threads
__global__ void __launch_bounds__(256) bwd_wv_part_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const int d = a.d;
  float* xs = sm;           // [32][d]
  float* gt = sm + 32 * d;  // [32][d]
  if (read_status(&a.hdr->status) != 0) return;
  const long long nrows = (long long)a.R * a.k;
  const long long r0 = (long long)blockIdx.x * kWvRows;
  const long long r1 = min(nrows, r0 + kWvRows);
  const int e = threadIdx.x % d, cg = threadIdx.x / d, cs = blockDim.x / d;
  const int nacc = d / cs;  // 64 (d=128) or 16 (d=64)
  float acc[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = 0.f;
  for (long long rb = r0; rb < r1; rb += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * d; i += blockDim.x) {
      const long long r = rb + i / d;
      const int c = i % d;
      float xv = 0.f, gv = 0.f;
      if (r < r1) {
        const long long u = r / a.k, j = r % a.k;
        xv = a.xsketch[(size_t)r * d + c];
        gv = a.Gt[((size_t)u * a.k_pad + j) * d + c];
      }
      xs[i] = xv;
      gt[i] = gv;
    }
    __syncthreads();
    for (int rr = 0; rr < 32; ++rr) {
      const float g = gt[rr * d + e];
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (i < nacc) acc[i] = fmaf(xs[rr * d + cg + cs * i], g, acc[i]);
    }
  }
  for (int i = 0; i < nacc; ++i)
    a.wv_part[((size_t)blockIdx.x * d + cg + cs * i) * d + e] = acc[i];
}

// ---- finish: dWv = sum of chunks; dP = dPn Wk / sqrt(d); dWk = dPn^T P / sqrt(d).
// 256 threads; lane l covers the columns l + 32 q (q < d / 32), so each thread carries
// d / 32 independent sums and loads. blockIdx.y = 0: dWv row blockIdx.x, the 8 warps
// taking the chunks in turn; 1: dWk row blockIdx.x, the warps splitting the prototypes;
// 2: dP rows 8 blockIdx.x + warp. Partial sums across warps are added in warp order.
template <typename TIn>
__global__ void __launch_bounds__(256) bwd_finish_kernel(BwdArgs a, const TIn* __restrict__ P,
                                                          const TIn* __restrict__ Wk, int nchunks,
                                                          float inv_sqrt_d) {
  if (read_status(&a.hdr->status) != 0) return;
  __shared__ float red[8][128];
  const int d = a.d, nq = d / 32;
  const int which = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (which == 2) {
    const int j = blockIdx.x * 8 + warp;
    if (j >= a.k) return;
#pragma unroll 4
    for (int c = 0; c < d; ++c) {
      const float g = a.dpp[(size_t)j * d + c];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq) acc[q] = fmaf(g, ldf(Wk, (size_t)c * d + lane + 32 * q), acc[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q < nq) a.dP[(size_t)j * d + lane + 32 * q] = acc[q] * inv_sqrt_d;
    return;
  }
  const int row = blockIdx.x;
  if (row >= d) return;  // uniform over the block
  if (which == 0) {
    for (int ch = warp; ch < nchunks; ch += 8)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq) acc[q] += a.wv_part[((size_t)ch * d + row) * d + lane + 32 * q];
  } else {
    const int per = (a.k + 7) / 8, j0 = warp * per, j1 = min(a.k, j0 + per);
#pragma unroll 4
    for (int j = j0; j < j1; ++j) {
      const float g = a.dpp[(size_t)j * d + row];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq) acc[q] = fmaf(g, ldf(P, (size_t)j * d + lane + 32 * q), acc[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q < nq) red[warp][lane + 32 * q] = acc[q];
  __syncthreads();
  if ((int)threadIdx.x < d) {
    float v = 0.f;
    for (int w = 0; w < 8; ++w) v += red[w][threadIdx.x];
    if (which == 0)
      a.dWv[(size_t)row * d + threadIdx.x] = v;
    else
      a.dWk[(size_t)row * d + threadIdx.x] = v * inv_sqrt_d;
  }
}

}  // namespace

size_t bwd_wv_chunks(int R, int k) {
  const long long n = (long long)R * k;
  return (size_t)((n + kWvRows - 1) / kWvRows);
}

// Launch sequence. The token kernel needs one block per tile; the tile count lives on
// the device, so the grid is the host's upper bound and surplus blocks exit.
template <typename TIn>
static cudaError_t launch_all(const BwdArgs& a, cudaStream_t s);

cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t s) {
  return a.dt == SA_BF16 ? launch_all<__nv_bfloat16>(a, s) : launch_all<float>(a, s);
}

template <typename TIn>
static cudaError_t launch_prep(const BwdArgs& a, cudaStream_t s) {
  if (a.R == 0) return cudaSuccess;
  const int d = a.d;
  // W_v is staged only when this kernel forms Gh itself (no Gtlo)
  const size_t smem = (size_t)((a.Gtlo ? 0 : d * (d + 1)) + kCP * d) * sizeof(float);
  cudaError_t e =
      cudaFuncSetAttribute(bwd_prep_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  bwd_prep_kernel<TIn><<<dim3((unsigned)a.R, (unsigned)(a.k_pad / kCP)), 256, smem, s>>>(
      a, static_cast<const TIn*>(a.Wv));
  return cudaGetLastError();
}

// dPn = sum of a.G partials (fixed order), dW_v chunks (unless wv_parts partials are
// already in a.wv_part), then dW_v, dP, dW_k.
template <typename TIn>
static cudaError_t launch_tail(const BwdArgs& a, int wv_parts, cudaStream_t s) {
  cudaError_t e;
  const int d = a.d;
  bwd_reduce_dpp_kernel<<<256, 256, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nch = wv_parts > 0 ? wv_parts : (int)bwd_wv_chunks(a.R, a.k);
  if (wv_parts == 0 && nch > 0) {
    const size_t smem_w = (size_t)(64 * d) * sizeof(float);
    bwd_wv_part_kernel<<<(unsigned)nch, 256, smem_w, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int fx = d > (a.k + 7) / 8 ? d : (a.k + 7) / 8;  // d rows of dWv / dWk, k / 8 of dP
  bwd_finish_kernel<TIn><<<dim3((unsigned)fx, 3), 256, 0, s>>>(
      a, static_cast<const TIn*>(a.P), static_cast<const TIn*>(a.Wk), nch, 1.0f / sqrtf((float)d));
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep(const BwdArgs& a, cudaStream_t s) {
  return a.dt == SA_BF16 ? launch_prep<__nv_bfloat16>(a, s) : launch_prep<float>(a, s);
}

cudaError_t launch_bwd_tail(const BwdArgs& a, int wv_parts, cudaStream_t s) {
  return a.dt == SA_BF16 ? launch_tail<__nv_bfloat16>(a, wv_parts, s)
                         : launch_tail<float>(a, wv_parts, s);
}

template <typename TIn>
static cudaError_t launch_all(const BwdArgs& a, cudaStream_t s) {
  cudaError_t e;
  const int d = a.d;
  const TIn* X = static_cast<const TIn*>(a.X);
  if ((e = launch_prep<TIn>(a, s)) != cudaSuccess) return e;
  if (a.n_total > 0) {
    const long long max_tiles = a.n_total / kTileTokens + a.R + 1;
    const size_t smem_t =
        (size_t)((kTileTokens + 2 * kCP) * (d + 1) + 2 * kTileTokens * 33 + kCP) * sizeof(float);
    e = cudaFuncSetAttribute(bwd_token_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_t);
    if (e != cudaSuccess) return e;
    bwd_token_kernel<TIn><<<(unsigned)max_tiles, 256, smem_t, s>>>(a, X);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const size_t smem_p = (size_t)((kTileTokens + 2 * kCP) * (d + 1) + kCP * 129 + 2 * kTileTokens + kCP) *
                          sizeof(float);
    e = cudaFuncSetAttribute(bwd_proto_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_p);
    if (e != cudaSuccess) return e;
    bwd_proto_kernel<TIn><<<dim3((unsigned)a.G, (unsigned)(a.k_pad / kCP)), 256, smem_p, s>>>(a, X);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return launch_tail<TIn>(a, 0, s);
}

}  // namespace sa
