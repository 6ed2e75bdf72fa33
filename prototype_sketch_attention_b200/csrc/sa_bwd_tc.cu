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
// Every contraction over d, k or the tokens runs as a tensor-core GEMM
// (sa_gemm_sm100.cu) with the elementwise work fused into its epilogue. D_t uses
// sum_j A_jt dA_jt = X_t . Y_t - sum_j A_jt c_j with Y = A Gh (which dX needs anyway), so
// dS comes straight out of one GEMM epilogue and no fp32 token x prototype matrix exists:
//   prep (CUDA cores)   Gt (fp32, bf16), bf16 Gh, c per user; bf16 U
//   fold                pn2 = bf16(Pn log2 e), pnn = bf16(Pn)
//   [lse not given]     GEMM S2 = X pn2^T -> per-tile log2-sum-exp -> lse2 per token
//   GEMM (user tiles)   A = 2^(X pn2^T - lse2) (bf16) and per-tile sums of A c_u
//   GEMM (user tiles)   Y = A Gh_u                                     fp32 [n, d]
//   CUDA cores          D_t = X_t . Y_t - sum_j A_jt c_j
//   GEMM (user tiles)   dS = A (X Gh_u^T - c_u - D_t)                  bf16 [n, k_pad]
//   GEMM (user tiles)   dX = dS pnn + Y
//   GEMM (split-K)      partials of dPn = dS^T X over token ranges
//   GEMM (split-K)      partials of dW_v = U^T Gt over (user, prototype) rows
//   tail (CUDA cores)   sums of the partials (fixed order), dP, dW_k
// 10 k d FLOP per token on the tensor cores (12 when the lse is recomputed).
#include <cmath>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// D_t = X_t . Y_t - sum of the row's per-tile partials of sum_j A_jt c_j.
// One warp per token row.
__global__ void __launch_bounds__(256) bwd_d_kernel(const __nv_bfloat16* __restrict__ X,
                                                    const float* __restrict__ Y, int d,
                                                    const float* __restrict__ cpart, int ntiles,
                                                    long long n_total, float* __restrict__ D,
                                                    const WsHeader* hdr) {
  if (read_status(&hdr->status) != 0) return;
  const int lane = threadIdx.x & 31;
  const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long t = w0; t < n_total; t += nw) {
    float acc = 0.f;
    for (int c = lane * 4; c < d; c += 128) {
      const float4 y = *reinterpret_cast<const float4*>(Y + t * d + c);
      const uint2 xv = *reinterpret_cast<const uint2*>(X + t * d + c);
      acc = fmaf(__uint_as_float(xv.x << 16), y.x, acc);
      acc = fmaf(__uint_as_float(xv.x & 0xFFFF0000u), y.y, acc);
      acc = fmaf(__uint_as_float(xv.y << 16), y.z, acc);
      acc = fmaf(__uint_as_float(xv.y & 0xFFFF0000u), y.w, acc);
    }
    for (int i = lane; i < ntiles; i += 32) acc -= cpart[t * ntiles + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) D[t] = acc;
  }
}

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

// Split-K count of the dPn GEMM: about two CTAs per SM, at most one split per K tile.
int bwd_tc_splits(int sms, int k_pad, int d, long long n_total) {
  const int tiles = (k_pad / 128) * ((d + 127) / 128);
  const long long kt = (n_total + 63) / 64;
  long long s = (2LL * sms + tiles - 1) / tiles;
  if (s > kt) s = kt;
  if (s < 1) s = 1;
  return (int)s;
}

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
  const int ntiles = k_pad / 128;
  const int nparts = 2 * ntiles;  // per-row partials: two column halves per tile
  if ((e = launch_bwd_prep(b, s)) != cudaSuccess) return e;
  const float isd = 1.0f / std::sqrt((float)d);
  if ((e = launch_fold(b.P, b.Wk, SA_BF16, k, k_pad, d, kLog2e * isd, a.pn2, true, s)) != cudaSuccess)
    return e;
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
    t.user_mode = 0;
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
    e = cudaMemsetAsync(b.dpp_part, 0, (size_t)a.splits * k_pad * d * sizeof(float), s);
    if (e != cudaSuccess) return e;
    return launch_bwd_tail(b, wv_parts, s);
  }
  const int m_plain = (int)((n + 127) / 128);
  const int m_user = (int)(n / 128 + R + 1);
  const GemmOperandDesc X_k = op(b.X, (uint64_t)n, (uint64_t)d, false);       // [n][d], K = d
  const GemmOperandDesc pn2_k = op(a.pn2, (uint64_t)k_pad, (uint64_t)d, false);
  const GemmOperandDesc gh_k = op(b.Ghb, (uint64_t)R * k_pad, (uint64_t)d, false);
  const GemmOperandDesc gh_mn = op(b.Ghb, (uint64_t)R * k_pad, (uint64_t)d, true);

  GemmArgs g = {};
  g.hdr = b.hdr;
  g.tile_start = b.tile_start;
  g.offsets = b.offsets;
  g.R = R;
  g.k_pad = k_pad;
  g.k_valid = k;
  g.splits = 1;

  // lse2 per token (log2 units): the forward's lse, or recomputed here
  const float* lse_src = a.lse;
  float lse_scale = kLog2e;
  if (!lse_src) {
    GemmArgs l = g;
    l.phases = 1;
    l.a[0] = X_k;
    l.b[0] = pn2_k;
    l.k_tiles[0] = (d + 63) / 64;
    l.user_mode = 0;
    l.M = (int)n;
    l.N = k_pad;
    l.m_tiles_bound = m_plain;
    l.epi = kEpiLse;
    l.dpart = a.dpart;
    l.dpart_ld = nparts;
    if ((e = launch_gemm(l, s)) != cudaSuccess) return e;
    bwd_lse_kernel<<<1024, 256, 0, s>>>(a.dpart, nparts, n, a.lse2, b.hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    lse_src = a.lse2;
    lse_scale = 1.f;
  }
  {  // A = 2^(X pn2^T - lse2), and per-tile sums of A c_u
    GemmArgs t = g;
    t.phases = 1;
    t.a[0] = X_k;
    t.b[0] = pn2_k;
    t.k_tiles[0] = (d + 63) / 64;
    t.user_mode = 1;
    t.N = k_pad;
    t.m_tiles_bound = m_user;
    t.epi = kEpiAExp;
    t.out_bf16 = a.A;
    t.ld_out = k_pad;
    t.lse2 = lse_src;
    t.lse_scale = lse_scale;
    t.c_user = b.cj;
    t.dpart = a.dpart;
    t.dpart_ld = nparts;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  {  // Y = A Gh_u
    GemmArgs t = g;
    t.phases = 1;
    t.a[0] = op(a.A, (uint64_t)n, (uint64_t)k_pad, false);
    t.b[0] = gh_mn;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = k_pad / 64;
    t.user_mode = 1;
    t.N = d;
    t.m_tiles_bound = m_user;
    t.epi = kEpiStoreF32;
    t.out_f32 = a.Y;
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  bwd_d_kernel<<<2048, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(b.X), a.Y, d, a.dpart, nparts,
                                    n, a.D, b.hdr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {  // dS = A (X Gh_u^T - c_u - D)
    GemmArgs t = g;
    t.phases = 1;
    t.a[0] = X_k;
    t.b[0] = gh_k;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = (d + 63) / 64;
    t.user_mode = 1;
    t.N = k_pad;
    t.m_tiles_bound = m_user;
    t.epi = kEpiDS;
    t.out_bf16 = a.dS;
    t.ld_out = k_pad;
    t.a_in = a.A;
    t.ld_a_in = k_pad;
    t.c_user = b.cj;
    t.drow = a.D;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  {  // dX = dS pnn + Y
    GemmArgs t = g;
    t.phases = 1;
    t.a[0] = op(a.dS, (uint64_t)n, (uint64_t)k_pad, false);
    t.b[0] = op(a.pnn, (uint64_t)k_pad, (uint64_t)d, true);
    t.k_tiles[0] = k_pad / 64;
    t.user_mode = 1;
    t.N = d;
    t.m_tiles_bound = m_user;
    t.epi = kEpiStoreF32;
    t.out_f32 = b.dX;
    t.ld_out = d;
    t.add_in = a.Y;
    t.ld_add = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  {  // dPn partials = dS^T X, split over token ranges
    GemmArgs t = g;
    t.phases = 1;
    t.a[0] = op(a.dS, (uint64_t)n, (uint64_t)k_pad, true);
    t.b[0] = op(b.X, (uint64_t)n, (uint64_t)d, true);
    t.k_tiles[0] = (int)((n + 63) / 64);
    t.user_mode = 0;
    t.M = k_pad;
    t.N = d;
    t.m_tiles_bound = ntiles;
    t.splits = a.splits;
    t.epi = kEpiStoreF32;
    t.out_f32 = b.dpp_part;
    t.ld_out = d;
    t.split_stride = (long long)k_pad * d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  return launch_bwd_tail(b, wv_parts, s);
}

}  // namespace sa
