// Candidate-to-sketch cross attention (the sketch branch of STCA) on the tensor cores.
//
// User u has a sketch S_u [k, d] (Sketch Attention's output) and candidates Q_c,
// c in [coff[u], coff[u+1]); every candidate of the user reads that one sketch:
//   out_c = sum_j softmax_j( (Q_c W_q) . (S_uj W_K) / sqrt(d) ) S_uj W_V
// ("100,000 videos in your pocket" blog, sections "2. STCA reasons at two time scales",
// the sketch branch, and "3. The system makes it cheap enough to matter", multi-request
// user-level batching). Refold: with Q' = Q (W_q W_K^T) log2(e) / sqrt(d) the scores are
// Q' S_u^T in log2 units, keys and values are the same matrix S_u, and W_V is applied
// once per candidate after the weighted sum. Steps, all on one stream:
//   1. schedule over the candidate offsets (128-candidate tiles that never span users)
//   2. S -> bf16 [R, k_pad, d] (zero rows past k); M^T = W_K W_q^T; Q' = Q M
//   3. per-candidate log2-sum-exp2 of Q' S_u^T: GEMM (kEpiLse partials) + combine
//   4. A = 2^(Q' S_u^T - lse2) in bf16 (GEMM, kEpiAExp), then O = A S_u in fp32
//   5. out = O W_V, with O entering as bf16 hi + lo (two accumulated GEMM phases)
#include <cmath>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kLn2F = 0.6931471805599453f;

// S (fp32 [R, k, d]) as bf16 [R, k_pad, d]; rows k..k_pad-1 of every user are zero.
__global__ void stca_sketch_bf16_kernel(const float* __restrict__ S, int R, int k, int k_pad,
                                        int d, __nv_bfloat16* __restrict__ Sb) {
  const long long n = (long long)R * k_pad * d;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i % d, rj = i / d, j = rj % k_pad, u = rj / k_pad;
    Sb[i] = __float2bfloat16_rn(j < k ? S[(u * k + j) * d + e] : 0.f);
  }
}

// lse2_c = log2 of the sum over the row's partials of 2^(partial); lse_c (natural log,
// nullable) = lse2_c ln 2. One thread per candidate.
__global__ void stca_lse_kernel(const float* __restrict__ dpart, int nparts, long long n,
                                float* __restrict__ lse2, float* __restrict__ lse,
                                const WsHeader* hdr) {
  if (read_status(&hdr->status) != 0) return;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < n;
       c += (long long)gridDim.x * blockDim.x) {
    const float* p = dpart + c * nparts;
    float m = -INFINITY;
    for (int i = 0; i < nparts; ++i) m = fmaxf(m, p[i]);
    float z = 0.f;
    for (int i = 0; i < nparts; ++i) z += ex2_approx(p[i] - m);
    const float l2 = m + lg2_approx(z);
    lse2[c] = l2;
    if (lse) lse[c] = l2 * kLn2F;
  }
}

// o = hi + lo with hi = bf16(o) and lo = bf16(o - hi): about 16 significant bits.
__global__ void stca_split_kernel(const float* __restrict__ O, long long n,
                                  __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const float v = O[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

GemmOperandDesc opd(const void* base, uint64_t rows, uint64_t cols, bool mn_major) {
  GemmOperandDesc o;
  o.base = base;
  o.rows = rows;
  o.cols = cols;
  o.mn_major = mn_major;
  return o;
}

}  // namespace

size_t stca_plan(int R, long long n_cand, int k, int d, StcaPlan* p) {
  StcaPlan q;
  q.k_pad = (k + 127) / 128 * 128;
  q.nparts = 2 * (q.k_pad / 128);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 255) / 256 * 256;
    return at;
  };
  const size_t n = (size_t)n_cand;
  q.hdr = take(sizeof(WsHeader));
  q.ts = take((size_t)(R + 1) * sizeof(long long));
  q.sb = take((size_t)R * q.k_pad * d * 2);
  q.mt = take((size_t)d * d * 2);
  q.qp = take(n * d * 2);
  q.dpart = take(n * q.nparts * sizeof(float));
  q.lse2 = take(n * sizeof(float));
  q.ab = take(n * q.k_pad * 2);
  q.o = take(n * d * sizeof(float));
  q.ohi = take(n * d * 2);
  q.olo = take(n * d * 2);
  q.total = o;
  *p = q;
  return o;
}

cudaError_t launch_stca_forward(const StcaArgs& a, cudaStream_t s) {
  const StcaPlan& p = a.plan;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + p.hdr);
  long long* ts = reinterpret_cast<long long*>(ws + p.ts);
  auto* Sb = reinterpret_cast<__nv_bfloat16*>(ws + p.sb);
  auto* Mt = reinterpret_cast<__nv_bfloat16*>(ws + p.mt);
  auto* Qp = reinterpret_cast<__nv_bfloat16*>(ws + p.qp);
  auto* dpart = reinterpret_cast<float*>(ws + p.dpart);
  auto* lse2 = reinterpret_cast<float*>(ws + p.lse2);
  auto* Ab = reinterpret_cast<__nv_bfloat16*>(ws + p.ab);
  auto* O = reinterpret_cast<float*>(ws + p.o);
  auto* Ohi = reinterpret_cast<__nv_bfloat16*>(ws + p.ohi);
  auto* Olo = reinterpret_cast<__nv_bfloat16*>(ws + p.olo);
  const int R = a.R, k = a.k, d = a.d, k_pad = p.k_pad;
  const long long n = a.n_cand;
  cudaError_t e;

  if ((e = launch_schedule(a.coff, R, n, hdr, ts, s)) != cudaSuccess) return e;
  if (n == 0) return cudaSuccess;
  stca_sketch_bf16_kernel<<<1024, 256, 0, s>>>(a.S, R, k, k_pad, d, Sb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // M^T = W_K W_q^T, then Q' = Q (M^T)^T log2(e) / sqrt(d) = Q W_q W_K^T log2(e) / sqrt(d)
  if ((e = launch_fold(a.WK, a.Wq, SA_BF16, d, d, d, 1.0f, Mt, true, s)) != cudaSuccess) return e;
  if ((e = launch_fold(a.Q, Mt, SA_BF16, (int)n, (int)n, d, kLog2eF / std::sqrt((float)d), Qp,
                       true, s)) != cudaSuccess)
    return e;

  GemmArgs g = {};
  g.hdr = hdr;
  g.tile_start = ts;
  g.offsets = a.coff;
  g.R = R;
  g.k_pad = k_pad;
  g.k_valid = k;
  g.splits = 1;
  g.phases = 1;
  g.user_mode = 1;
  g.m_tiles_bound = (int)(n / 128 + R + 1);
  const GemmOperandDesc qp_k = opd(Qp, (uint64_t)n, (uint64_t)d, false);
  const GemmOperandDesc sb_k = opd(Sb, (uint64_t)R * k_pad, (uint64_t)d, false);
  const GemmOperandDesc sb_mn = opd(Sb, (uint64_t)R * k_pad, (uint64_t)d, true);
  {  // per-candidate log2-sum-exp2 partials of the scores over each 64-row half tile
    GemmArgs t = g;
    t.a[0] = qp_k;
    t.b[0] = sb_k;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = (d + 63) / 64;
    t.N = k_pad;
    t.epi = kEpiLse;
    t.dpart = dpart;
    t.dpart_ld = p.nparts;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  stca_lse_kernel<<<1024, 256, 0, s>>>(dpart, p.nparts, n, lse2, a.lse, hdr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {  // A = 2^(Q' S_u^T - lse2), the attention weights (each row sums to 1)
    GemmArgs t = g;
    t.a[0] = qp_k;
    t.b[0] = sb_k;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = (d + 63) / 64;
    t.N = k_pad;
    t.epi = kEpiAExp;
    t.out_bf16 = Ab;
    t.ld_out = k_pad;
    t.lse2 = lse2;
    t.lse_scale = 1.f;
    t.c_user = nullptr;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  {  // O = A S_u: the same sketch rows, now as values
    GemmArgs t = g;
    t.a[0] = opd(Ab, (uint64_t)n, (uint64_t)k_pad, false);
    t.b[0] = sb_mn;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = k_pad / 64;
    t.N = d;
    t.epi = kEpiStoreF32;
    t.out_f32 = O;
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  stca_split_kernel<<<1024, 256, 0, s>>>(O, n * d, Ohi, Olo);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {  // out = (hi + lo) W_V
    GemmArgs t = {};
    t.hdr = hdr;
    t.a[0] = opd(Ohi, (uint64_t)n, (uint64_t)d, false);
    t.a[1] = opd(Olo, (uint64_t)n, (uint64_t)d, false);
    t.b[0] = opd(a.WV, (uint64_t)d, (uint64_t)d, true);  // W_V[f][e]: rows = K, cols = N
    t.b[1] = t.b[0];
    t.phases = 2;
    t.k_tiles[0] = t.k_tiles[1] = d / 64;
    t.user_mode = 0;
    t.M = (int)n;
    t.N = d;
    t.m_tiles_bound = (int)((n + 127) / 128);
    t.splits = 1;
    t.epi = kEpiStoreF32;
    t.out_f32 = a.out;
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sa
