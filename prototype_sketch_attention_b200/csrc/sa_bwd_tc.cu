// Sketch Attention backward on tcgen05 tensor cores (bf16 inputs, fp32 accumulate).
//
// The gradient of the sketch (blog "100,000 videos in your pocket", section "1. Sketch
// Attention compresses the history": the compression is differentiable) with
// Pn = P W_k^T / sqrt(d), G = dL/dsketch, Gm = dL/dmass and, per user u,
//   Gt = G / mass,  Gh = Gt W_v^T,  c_j = Gt_j . sketch_j - Gm_j,
//   A_jt = exp(Pn_j . X_t - lse_t),  dA_jt = Gh_j . X_t - c_j,
//   D_t = sum_j A_jt dA_jt,  dS_jt = A_jt (dA_jt - D_t),
//   dX_t = sum_j dS_jt Pn_j + sum_j A_jt Gh_j,   dPn = sum_t dS_t^T X_t,
// then dP = dPn W_k / sqrt(d), dW_k = dPn^T P / sqrt(d), dW_v = sum_u U_u^T Gt_u.
//
// Launch sequence (bf16):
//   prep (CUDA cores)   Gt (fp32, and bf16 hi + lo parts), c per user
//   GEMM                bf16 Gh = (Gt_hi + Gt_lo) W_v^T for every user (two phases)
//   fold                pnn = bf16(Pn)  [and pn2 = bf16(Pn log2 e) when the lse is recomputed]
//   GEMM (split-K)      partials of dW_v = U^T Gt over (user, prototype) rows (bf16 U)
//   [lse not given]     GEMM S2 = X pn2^T -> per-tile log2-sum-exp -> lse2 per token
//   memset dX; the single-pass kernel (sa_bwd_fused.cu): A, dA, D, dS per tile in
//                       shared memory and TMEM, dX partials added in L2, dPn per cluster
//   tail (CUDA cores)   sums of the partials (fixed order), dP, dW_k
// 10 k d FLOP per token on the tensor cores (12 when the lse is recomputed).
#include <cmath>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// U (the forward's xsketch, fp32 [R, k, d]) as bf16 [R, k_pad, d] with zero padding rows.
__global__ void bwd_u_bf16_kernel(const float* __restrict__ U, int R, int k, int k_pad, int d,
                                  __nv_bfloat16* __restrict__ Ub) {
  const long long n = (long long)R * k_pad * d;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i % d, rj = i / d, j = rj % k_pad, u = rj / k_pad;
    Ub[i] = __float2bfloat16_rn(j < k ? U[(u * k + j) * d + e] : 0.f);
  }
}

// lse2_t = log2 sum over the row's tiles of 2^(partial).  One thread per token.
__global__ void bwd_lse_kernel(const float* __restrict__ dpart, int ntiles, long long n_total,
                               float* __restrict__ lse2, const WsHeader* hdr) {
  if (read_status(&hdr->status) != 0) return;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n_total;
       t += (long long)gridDim.x * blockDim.x) {
    const float* p = dpart + t * ntiles;
    float m = -INFINITY;
    for (int i = 0; i < ntiles; ++i) m = fmaxf(m, p[i]);
    float z = 0.f;
    for (int i = 0; i < ntiles; ++i) z += ex2_approx(p[i] - m);
    lse2[t] = m + lg2_approx(z);
  }
}

GemmOperandDesc op(const void* base, uint64_t rows, uint64_t cols, bool mn_major) {
  GemmOperandDesc o;
  o.base = base;
  o.rows = rows;
  o.cols = cols;
  o.mn_major = mn_major;
  return o;
}

}  // namespace

// Split-K count of the dW_v GEMM (one 128 x 128 output tile): about two CTAs per SM.
int bwd_tc_wv_splits(int sms, int R, int k_pad) {
  const long long kt = ((long long)R * k_pad + 63) / 64;
  long long s = 2LL * sms;
  if (s > kt) s = kt;
  if (s < 1) s = 1;
  return (int)s;
}

cudaError_t launch_bwd_tc(const BwdTcArgs& a, cudaStream_t s) {
  const BwdArgs& b = a.b;
  cudaError_t e;
  const int d = b.d, k = b.k, k_pad = b.k_pad, R = b.R;
  const long long n = b.n_total;
  const int nparts = 2 * (k_pad / 128);  // per-row lse partials: two column halves per tile
  if ((e = launch_bwd_prep(b, s)) != cudaSuccess) return e;
  if (R > 0) {  // Gh = Gt W_v^T for every user: (Gt_hi + Gt_lo) W_v^T, two accumulated phases
    GemmArgs t = {};
    t.hdr = b.hdr;
    t.phases = 2;
    t.a[0] = op(b.Gtb, (uint64_t)R * k_pad, (uint64_t)d, false);
    t.b[0] = op(b.Wv, (uint64_t)d, (uint64_t)d, false);
    t.a[1] = op(b.Gtlo, (uint64_t)R * k_pad, (uint64_t)d, false);
    t.b[1] = op(b.Wv, (uint64_t)d, (uint64_t)d, false);
    t.k_tiles[0] = t.k_tiles[1] = (d + 63) / 64;
    t.M = R * k_pad;
    t.N = d;
    t.m_tiles_bound = (R * k_pad + 127) / 128;
    t.splits = 1;
    t.epi = kEpiStoreBf16;
    t.out_bf16 = b.Ghb;
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  const float isd = 1.0f / std::sqrt((float)d);
  if ((e = launch_fold(b.P, b.Wk, SA_BF16, k, k_pad, d, isd, a.pnn, true, s)) != cudaSuccess)
    return e;
  if (R > 0) {  // dW_v = sum over (user, prototype) rows of U^T Gt, split-K
    bwd_u_bf16_kernel<<<1024, 256, 0, s>>>(b.xsketch, R, k, k_pad, d, a.Ub);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    GemmArgs t = {};
    t.hdr = b.hdr;
    t.phases = 1;
    t.a[0] = op(a.Ub, (uint64_t)R * k_pad, (uint64_t)d, true);
    t.b[0] = op(b.Gtb, (uint64_t)R * k_pad, (uint64_t)d, true);
    t.k_tiles[0] = (int)(((long long)R * k_pad + 63) / 64);
    t.M = d;
    t.N = d;
    t.m_tiles_bound = 1;
    t.splits = a.wv_splits;
    t.epi = kEpiStoreF32;
    t.out_f32 = b.wv_part;
    t.ld_out = d;
    t.split_stride = (long long)d * d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  } else {
    e = cudaMemsetAsync(b.wv_part, 0, (size_t)d * d * sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  const int wv_parts = R > 0 ? a.wv_splits : 1;
  if (n == 0) {
    e = cudaMemsetAsync(b.dpp_part, 0, (size_t)b.G * k_pad * d * sizeof(float), s);
    if (e != cudaSuccess) return e;
    return launch_bwd_tail(b, wv_parts, s);
  }
  // lse2 per token (log2 units): the forward's lse, or recomputed here
  const float* lse_src = a.lse;
  float lse_scale = kLog2e;
  if (!lse_src) {
    if ((e = launch_fold(b.P, b.Wk, SA_BF16, k, k_pad, d, kLog2e * isd, a.pn2, true, s)) != cudaSuccess)
      return e;
    GemmArgs l = {};
    l.hdr = b.hdr;
    l.k_valid = k;
    l.splits = 1;
    l.phases = 1;
    l.a[0] = op(b.X, (uint64_t)n, (uint64_t)d, false);
    l.b[0] = op(a.pn2, (uint64_t)k_pad, (uint64_t)d, false);
    l.k_tiles[0] = (d + 63) / 64;
    l.M = (int)n;
    l.N = k_pad;
    l.m_tiles_bound = (int)((n + 127) / 128);
    l.epi = kEpiLse;
    l.dpart = a.dpart;
    l.dpart_ld = nparts;
    if ((e = launch_gemm(l, s)) != cudaSuccess) return e;
    bwd_lse_kernel<<<1024, 256, 0, s>>>(a.dpart, nparts, n, a.lse2, b.hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    lse_src = a.lse2;
    lse_scale = 1.f;
  }
  // dX is the sum of the C prototype slices' partials, which the fused kernel adds in L2
  if ((e = cudaMemsetAsync(b.dX, 0, (size_t)n * d * sizeof(float), s)) != cudaSuccess) return e;
  BwdFusedArgs f;
  f.X = b.X;
  f.offsets = b.offsets;
  f.R = R;
  f.k_valid = k;
  f.C = a.C;
  f.k_pad = k_pad;
  f.d = d;
  f.G = a.G;
  f.n_total = n;
  f.hdr = b.hdr;
  f.tile_start = b.tile_start;
  f.pn = a.pnn;
  f.gh = b.Ghb;
  f.cj = b.cj;
  f.lse = lse_src;
  f.lse_scale = lse_scale;
  f.dX = b.dX;
  f.dpp_part = b.dpp_part;
  f.budget = kDefaultWaitBudget;
  if ((e = launch_bwd_fused(f, s)) != cudaSuccess) return e;
  return launch_bwd_tail(b, wv_parts, s);
}

}  // namespace sa
