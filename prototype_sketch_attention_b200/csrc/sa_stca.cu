// Candidate-to-sketch cross attention (the sketch branch of STCA) on the tensor cores.
//
// User u has a sketch S_u [k, d] (Sketch Attention's output) and candidates Q_c,
// c in [coff[u], coff[u+1]); every candidate of the user reads that one sketch:
//   out_c = sum_j softmax_j( (Q_c W_q) . (S_uj W_K) / sqrt(d) ) S_uj W_V
// ("100,000 videos in your pocket" blog, sections "2. STCA reasons at two time scales",
// the sketch branch, and "3. The system makes it cheap enough to matter", multi-request
// user-level batching). Refold: with Q' = Q (W_q W_K^T) log2(e) / sqrt(d) the scores are
// Q' S_u^T in log2 units, keys and values are the same matrix S_u, and W_V is applied
// once per candidate after the weighted sum.
// The forward is the flash kernel of the ragged-key attention (sa_stca_keys.cu) with the
// bf16 sketch as the key rows: S -> bf16 [R, k_pad, d], user u's keys the rows
// [u k_pad, u k_pad + k). The backward is composed from the tcgen05 GEMM, all on one
// stream:
//   1. schedule over the candidate offsets (128-candidate tiles that never span users)
//   2. S -> bf16 [R, k_pad, d] (zero rows past k); M^T = W_K W_q^T; Q' = Q M
//   3. per-candidate log2-sum-exp2 of Q' S_u^T: GEMM (kEpiLse partials) + combine
//   4. A = 2^(Q' S_u^T - lse2) in bf16 (GEMM, kEpiAExp), then O = A S_u in fp32
// and then, with G = dL/dout and natural-log units
// (z = Q M S_u^T / sqrt(d), M = W_q W_K^T):
//   dO = G W_V^T,  dW_V = O^T G,  D_c = dO_c . O_c,  dZ = A (dO S_u^T - D)
//   G1 = dZ S_u,  dQ = G1 M^T / sqrt(d),  dM = Q^T G1 / sqrt(d)
//   dW_q = dM W_K,  dW_K = dM^T W_q,  dS_u = dZ_u^T (Q_u M / sqrt(d)) + A_u^T dO_u
// dS_u is a sum over user u's candidates only, one GEMM per user (its candidates as K).
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

// User u's sketch rows within the bf16 sketch: [u k_pad, u k_pad + k).
__global__ void stca_sketch_ranges_kernel(int R, int k, int k_pad, int64_t* __restrict__ kb,
                                          int64_t* __restrict__ ke) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < R; u += gridDim.x * blockDim.x) {
    kb[u] = (int64_t)u * k_pad;
    ke[u] = (int64_t)u * k_pad + k;
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

__global__ void stca_to_bf16_kernel(const float* __restrict__ x, long long n,
                                    __nv_bfloat16* __restrict__ y) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

// D_c = dO_c . O_c, one warp per candidate.
__global__ void stca_rowdot_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                   long long n, int d, float* __restrict__ D) {
  const int lane = threadIdx.x & 31;
  const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long c = w0; c < n; c += nw) {
    float acc = 0.f;
    for (int e = lane; e < d; e += 32) acc = fmaf(a[c * d + e], b[c * d + e], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) D[c] = acc;
  }
}

// out[i] = scale * sum over s < parts of part[s][i] (split-K partials, in order).
__global__ void stca_sum_parts_kernel(const float* __restrict__ part, int parts, long long n,
                                      float scale, float* __restrict__ out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int q = 0; q < parts; ++q) v += part[(long long)q * n + i];
    out[i] = scale * v;
  }
}

// dW_q = dM W_K and dW_K = dM^T W_q for d x d matrices (fp32 dM, bf16 weights).
__global__ void stca_weight_grads_kernel(const float* __restrict__ dM,
                                         const __nv_bfloat16* __restrict__ Wq,
                                         const __nv_bfloat16* __restrict__ WK, int d,
                                         float* __restrict__ dWq, float* __restrict__ dWK) {
  const int r = blockIdx.x;
  for (int x = threadIdx.x; x < d; x += blockDim.x) {
    float gq = 0.f, gk = 0.f;
    for (int f = 0; f < d; ++f) {
      gq = fmaf(dM[r * d + f], __bfloat162float(WK[f * d + x]), gq);
      gk = fmaf(dM[f * d + r], __bfloat162float(Wq[f * d + x]), gk);
    }
    dWq[r * d + x] = gq;
    dWK[r * d + x] = gk;
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

size_t stca_plan(int R, long long n_cand, int k, int d, bool backward, int sms, StcaPlan* p) {
  StcaPlan q;
  q.k_pad = (k + 127) / 128 * 128;
  q.nparts = 2 * (q.k_pad / 128);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 255) / 256 * 256;
    return at;
  };
  if (!backward) {  // the flash kernel over each user's sketch rows
    StcaKeysPlan kp;
    o = stca_keys_plan(R, n_cand, d, false, 0, &kp);
    q.hdr = kp.hdr;
    q.sb = take((size_t)R * q.k_pad * d * 2);
    q.kb = take((size_t)R * sizeof(int64_t));
    q.ke = take((size_t)R * sizeof(int64_t));
    q.total = o;
    *p = q;
    return o;
  }
  const size_t n = (size_t)n_cand;
  const size_t nd = n * d;
  q.hdr = take(sizeof(WsHeader));
  q.ts = take((size_t)(R + 1) * sizeof(long long));
  q.sb = take((size_t)R * q.k_pad * d * 2);
  q.mt = take((size_t)d * d * 2);
  q.qp = take(nd * 2);
  q.dpart = take(n * q.nparts * sizeof(float));
  q.lse2 = take(n * sizeof(float));
  q.ab = take(n * q.k_pad * 2);
  q.o = take(nd * sizeof(float));
  q.ohi = take(nd * 2);
  q.olo = take(nd * 2);
  if (backward) {
    const long long kt = ((long long)n + 63) / 64;
    long long sp = 2LL * (sms > 0 ? sms : 148);
    if (sp > kt) sp = kt;
    q.splits = (int)(sp < 1 ? 1 : sp);
    q.mts = take((size_t)d * d * 2);
    q.qn = take(nd * 2);
    q.do_f = take(nd * sizeof(float));
    q.do_b = take(nd * 2);
    q.dd = take(n * sizeof(float));
    q.czero = take((size_t)R * q.k_pad * sizeof(float));
    q.dz = take(n * q.k_pad * 2);
    q.g1 = take(nd * sizeof(float));
    q.g1hi = take(nd * 2);
    q.g1lo = take(nd * 2);
    q.gb = take(nd * 2);
    q.ob = take(nd * 2);
    q.ghi = take(nd * 2);
    q.glo = take(nd * 2);
    q.part = take((size_t)q.splits * d * d * sizeof(float));
    q.dm = take((size_t)d * d * sizeof(float));
  }
  q.total = o;
  *p = q;
  return o;
}

namespace {

struct Bufs {
  WsHeader* hdr;
  long long* ts;
  __nv_bfloat16 *Sb, *Mt, *Qp, *Ab, *Ohi, *Olo;
  float *dpart, *lse2, *O;
};

Bufs bufs(const StcaPlan& p, void* workspace) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Bufs b;
  b.hdr = reinterpret_cast<WsHeader*>(ws + p.hdr);
  b.ts = reinterpret_cast<long long*>(ws + p.ts);
  b.Sb = reinterpret_cast<__nv_bfloat16*>(ws + p.sb);
  b.Mt = reinterpret_cast<__nv_bfloat16*>(ws + p.mt);
  b.Qp = reinterpret_cast<__nv_bfloat16*>(ws + p.qp);
  b.Ab = reinterpret_cast<__nv_bfloat16*>(ws + p.ab);
  b.Ohi = reinterpret_cast<__nv_bfloat16*>(ws + p.ohi);
  b.Olo = reinterpret_cast<__nv_bfloat16*>(ws + p.olo);
  b.dpart = reinterpret_cast<float*>(ws + p.dpart);
  b.lse2 = reinterpret_cast<float*>(ws + p.lse2);
  b.O = reinterpret_cast<float*>(ws + p.o);
  return b;
}

GemmArgs user_gemm(const StcaArgs& a, const Bufs& b) {
  GemmArgs g = {};
  g.hdr = b.hdr;
  g.tile_start = b.ts;
  g.offsets = a.coff;
  g.R = a.R;
  g.k_pad = a.plan.k_pad;
  g.k_valid = a.k;
  g.splits = 1;
  g.phases = 1;
  g.user_mode = 1;
  g.m_tiles_bound = (int)(a.n_cand / 128 + a.R + 1);
  return g;
}

// Steps 1-4: schedule, bf16 sketch, Q', lse2, A and O = A S_u. Needs n_cand > 0 after
// the schedule (the caller returns early otherwise).
cudaError_t forward_core(const StcaArgs& a, const Bufs& b, cudaStream_t s) {
  const int R = a.R, k = a.k, d = a.d, k_pad = a.plan.k_pad;
  const long long n = a.n_cand;
  cudaError_t e;
  stca_sketch_bf16_kernel<<<1024, 256, 0, s>>>(a.S, R, k, k_pad, d, b.Sb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // M^T = W_K W_q^T, then Q' = Q (M^T)^T log2(e) / sqrt(d) = Q W_q W_K^T log2(e) / sqrt(d)
  if ((e = launch_fold(a.WK, a.Wq, SA_BF16, d, d, d, 1.0f, b.Mt, true, s)) != cudaSuccess) return e;
  if ((e = launch_fold(a.Q, b.Mt, SA_BF16, (int)n, (int)n, d, kLog2eF / std::sqrt((float)d), b.Qp,
                       true, s)) != cudaSuccess)
    return e;
  const GemmArgs g = user_gemm(a, b);
  const GemmOperandDesc qp_k = opd(b.Qp, (uint64_t)n, (uint64_t)d, false);
  const GemmOperandDesc sb_k = opd(b.Sb, (uint64_t)R * k_pad, (uint64_t)d, false);
  const GemmOperandDesc sb_mn = opd(b.Sb, (uint64_t)R * k_pad, (uint64_t)d, true);
  {  // per-candidate log2-sum-exp2 partials of the scores over each 64-row half tile
    GemmArgs t = g;
    t.a[0] = qp_k;
    t.b[0] = sb_k;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = (d + 63) / 64;
    t.N = k_pad;
    t.epi = kEpiLse;
    t.dpart = b.dpart;
    t.dpart_ld = a.plan.nparts;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  stca_lse_kernel<<<1024, 256, 0, s>>>(b.dpart, a.plan.nparts, n, b.lse2, a.lse, b.hdr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {  // A = 2^(Q' S_u^T - lse2), the attention weights (each row sums to 1)
    GemmArgs t = g;
    t.a[0] = qp_k;
    t.b[0] = sb_k;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = (d + 63) / 64;
    t.N = k_pad;
    t.epi = kEpiAExp;
    t.out_bf16 = b.Ab;
    t.ld_out = k_pad;
    t.lse2 = b.lse2;
    t.lse_scale = 1.f;
    t.c_user = nullptr;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  {  // O = A S_u: the same sketch rows, now as values
    GemmArgs t = g;
    t.a[0] = opd(b.Ab, (uint64_t)n, (uint64_t)k_pad, false);
    t.b[0] = sb_mn;
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = k_pad / 64;
    t.N = d;
    t.epi = kEpiStoreF32;
    t.out_f32 = b.O;
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t stca_split_hilo(const float* x, long long n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                            cudaStream_t s) {
  stca_split_kernel<<<1024, 256, 0, s>>>(x, n, hi, lo);
  return cudaGetLastError();
}

cudaError_t stca_to_bf16(const float* x, long long n, __nv_bfloat16* y, cudaStream_t s) {
  stca_to_bf16_kernel<<<1024, 256, 0, s>>>(x, n, y);
  return cudaGetLastError();
}

cudaError_t stca_weight_grads(const float* dM, const void* Wq, const void* WK, int d, float* dWq,
                              float* dWK, cudaStream_t s) {
  stca_weight_grads_kernel<<<d, 128, 0, s>>>(dM, static_cast<const __nv_bfloat16*>(Wq),
                                             static_cast<const __nv_bfloat16*>(WK), d, dWq, dWK);
  return cudaGetLastError();
}

// out[n, N] = (hi + lo) B with B given as an operand descriptor (two accumulated phases).
cudaError_t gemm_hilo(const WsHeader* hdr, const __nv_bfloat16* hi, const __nv_bfloat16* lo,
                      long long n, int d, GemmOperandDesc bop, float* out, cudaStream_t s) {
  GemmArgs t = {};
  t.hdr = hdr;
  t.a[0] = opd(hi, (uint64_t)n, (uint64_t)d, false);
  t.a[1] = opd(lo, (uint64_t)n, (uint64_t)d, false);
  t.b[0] = bop;
  t.b[1] = bop;
  t.phases = 2;
  t.k_tiles[0] = t.k_tiles[1] = d / 64;
  t.user_mode = 0;
  t.M = (int)n;
  t.N = d;
  t.m_tiles_bound = (int)((n + 127) / 128);
  t.splits = 1;
  t.epi = kEpiStoreF32;
  t.out_f32 = out;
  t.ld_out = d;
  return launch_gemm(t, s);
}

// part[s] = A^T B over split s of the rows (both [n, d] bf16), then out = scale * sum.
cudaError_t gemm_tn_sum(const WsHeader* hdr, const __nv_bfloat16* A, const __nv_bfloat16* B,
                        long long n, int d, int splits, float* part, float scale, float* out,
                        cudaStream_t s) {
  GemmArgs t = {};
  t.hdr = hdr;
  t.phases = 1;
  t.a[0] = opd(A, (uint64_t)n, (uint64_t)d, true);
  t.b[0] = opd(B, (uint64_t)n, (uint64_t)d, true);
  t.k_tiles[0] = (int)((n + 63) / 64);
  t.user_mode = 0;
  t.M = d;
  t.N = d;
  t.m_tiles_bound = (d + 127) / 128;
  t.splits = splits;
  t.epi = kEpiStoreF32;
  t.out_f32 = part;
  t.ld_out = d;
  t.split_stride = (long long)d * d;
  cudaError_t e = cudaMemsetAsync(part, 0, (size_t)splits * d * d * sizeof(float), s);
  if (e != cudaSuccess) return e;
  if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  stca_sum_parts_kernel<<<(d * d + 255) / 256, 256, 0, s>>>(part, splits, (long long)d * d, scale,
                                                            out);
  return cudaGetLastError();
}

// The forward is the ragged-key attention (sa_stca_keys.cu) over each user's sketch rows:
// the sketch in bf16 [R, k_pad, d], user u's keys the rows [u k_pad, u k_pad + k).
cudaError_t launch_stca_forward(const StcaArgs& a, cudaStream_t s) {
  const StcaPlan& p = a.plan;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  __nv_bfloat16* Sb = reinterpret_cast<__nv_bfloat16*>(ws + p.sb);
  int64_t* kb = reinterpret_cast<int64_t*>(ws + p.kb);
  int64_t* ke = reinterpret_cast<int64_t*>(ws + p.ke);
  cudaError_t e;
  if (a.R > 0) {
    stca_sketch_bf16_kernel<<<1024, 256, 0, s>>>(a.S, a.R, a.k, p.k_pad, a.d, Sb);
    stca_sketch_ranges_kernel<<<(a.R + 255) / 256, 256, 0, s>>>(a.R, a.k, p.k_pad, kb, ke);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  StcaKeysArgs k;
  k.Q = a.Q;
  k.coff = a.coff;
  k.R = a.R;
  k.d = a.d;
  k.n_cand = a.n_cand;
  k.Kx = Sb;
  k.n_keys = (long long)a.R * p.k_pad;
  k.kb = kb;
  k.ke = ke;
  k.Wq = a.Wq;
  k.WK = a.WK;
  k.WV = a.WV;
  k.out = a.out;
  k.lse = a.lse;
  k.workspace = a.workspace;
  stca_keys_plan(a.R, a.n_cand, a.d, false, 0, &k.plan);
  return launch_stca_keys_forward(k, s);
}

cudaError_t launch_stca_backward(const StcaArgs& a, const StcaGrads& gr, cudaStream_t s) {
  const StcaPlan& p = a.plan;
  const Bufs b = bufs(p, a.workspace);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const int R = a.R, k = a.k, d = a.d, k_pad = p.k_pad;
  const long long n = a.n_cand;
  const float isd = 1.0f / std::sqrt((float)d);
  cudaError_t e;
  if ((e = launch_schedule(a.coff, R, n, b.hdr, b.ts, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(gr.dS, 0, (size_t)R * k * d * sizeof(float), s)) != cudaSuccess) return e;
  if (n == 0) {
    for (float* g : {gr.dWq, gr.dWK, gr.dWV})
      if ((e = cudaMemsetAsync(g, 0, (size_t)d * d * sizeof(float), s)) != cudaSuccess) return e;
    return cudaSuccess;
  }
  if ((e = forward_core(a, b, s)) != cudaSuccess) return e;
  // bf16 copies: O (for dW_V) and G = dL/dout as hi + lo (for dO) and as bf16 (for dW_V)
  stca_to_bf16_kernel<<<1024, 256, 0, s>>>(b.O, n * d, bf(p.ob));
  stca_split_kernel<<<1024, 256, 0, s>>>(gr.dout, n * d, bf(p.ghi), bf(p.glo));
  stca_to_bf16_kernel<<<1024, 256, 0, s>>>(gr.dout, n * d, bf(p.gb));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // dO = G W_V^T: B[n = f][k = e] = W_V[f][e], K-major
  if ((e = gemm_hilo(b.hdr, bf(p.ghi), bf(p.glo), n, d, opd(a.WV, (uint64_t)d, (uint64_t)d, false),
                     f32(p.do_f), s)) != cudaSuccess)
    return e;
  // dW_V = O^T G
  if ((e = gemm_tn_sum(b.hdr, bf(p.ob), bf(p.gb), n, d, p.splits, f32(p.part), 1.0f, gr.dWV, s)) !=
      cudaSuccess)
    return e;
  stca_to_bf16_kernel<<<1024, 256, 0, s>>>(f32(p.do_f), n * d, bf(p.do_b));
  stca_rowdot_kernel<<<1024, 256, 0, s>>>(f32(p.do_f), b.O, n, d, f32(p.dd));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(f32(p.czero), 0, (size_t)R * k_pad * sizeof(float), s)) != cudaSuccess)
    return e;
  const GemmArgs g = user_gemm(a, b);
  {  // dZ = A (dO S_u^T - D), bf16
    GemmArgs t = g;
    t.a[0] = opd(bf(p.do_b), (uint64_t)n, (uint64_t)d, false);
    t.b[0] = opd(b.Sb, (uint64_t)R * k_pad, (uint64_t)d, false);
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = (d + 63) / 64;
    t.N = k_pad;
    t.epi = kEpiDS;
    t.out_bf16 = bf(p.dz);
    t.ld_out = k_pad;
    t.a_in = b.Ab;
    t.ld_a_in = k_pad;
    t.c_user = f32(p.czero);
    t.drow = f32(p.dd);
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  {  // G1 = dZ S_u
    GemmArgs t = g;
    t.a[0] = opd(bf(p.dz), (uint64_t)n, (uint64_t)k_pad, false);
    t.b[0] = opd(b.Sb, (uint64_t)R * k_pad, (uint64_t)d, true);
    t.b_user_rows[0] = k_pad;
    t.k_tiles[0] = k_pad / 64;
    t.N = d;
    t.epi = kEpiStoreF32;
    t.out_f32 = f32(p.g1);
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  stca_split_kernel<<<1024, 256, 0, s>>>(f32(p.g1), n * d, bf(p.g1hi), bf(p.g1lo));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // dQ = G1 M^T / sqrt(d): Mts = M^T / sqrt(d) stored [f][r] is B MN-major (rows = K = f)
  if ((e = launch_fold(a.WK, a.Wq, SA_BF16, d, d, d, isd, bf(p.mts), true, s)) != cudaSuccess)
    return e;
  if ((e = gemm_hilo(b.hdr, bf(p.g1hi), bf(p.g1lo), n, d, opd(bf(p.mts), (uint64_t)d, (uint64_t)d,
                                                              true),
                     gr.dQ, s)) != cudaSuccess)
    return e;
  // dM = Q^T G1 / sqrt(d), then dW_q = dM W_K and dW_K = dM^T W_q
  stca_to_bf16_kernel<<<1024, 256, 0, s>>>(f32(p.g1), n * d, bf(p.gb));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = gemm_tn_sum(b.hdr, static_cast<const __nv_bfloat16*>(a.Q), bf(p.gb), n, d, p.splits,
                       f32(p.part), isd, f32(p.dm), s)) != cudaSuccess)
    return e;
  stca_weight_grads_kernel<<<d, 128, 0, s>>>(f32(p.dm), static_cast<const __nv_bfloat16*>(a.Wq),
                                             static_cast<const __nv_bfloat16*>(a.WK), d, gr.dWq,
                                             gr.dWK);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // Qn = Q M / sqrt(d) (the keys' side of the scores, natural units)
  if ((e = launch_fold(a.Q, b.Mt, SA_BF16, (int)n, (int)n, d, isd, bf(p.qn), true, s)) !=
      cudaSuccess)
    return e;
  // dS_u = dZ_u^T Qn_u + A_u^T dO_u: one GEMM per user with candidates, its rows as K
  for (int u = 0; u < R; ++u) {
    const long long c0 = gr.coff_host[u], nu = gr.coff_host[u + 1] - c0;
    if (nu <= 0) continue;
    GemmArgs t = {};
    t.hdr = b.hdr;
    t.phases = 2;
    t.a[0] = opd(bf(p.dz) + c0 * k_pad, (uint64_t)nu, (uint64_t)k_pad, true);
    t.b[0] = opd(bf(p.qn) + c0 * d, (uint64_t)nu, (uint64_t)d, true);
    t.a[1] = opd(b.Ab + c0 * k_pad, (uint64_t)nu, (uint64_t)k_pad, true);
    t.b[1] = opd(bf(p.do_b) + c0 * d, (uint64_t)nu, (uint64_t)d, true);
    t.k_tiles[0] = t.k_tiles[1] = (int)((nu + 63) / 64);
    t.user_mode = 0;
    t.M = k;
    t.N = d;
    t.m_tiles_bound = (k + 127) / 128;
    t.splits = 1;
    t.epi = kEpiStoreF32;
    t.out_f32 = gr.dS + (long long)u * k * d;
    t.ld_out = d;
    if ((e = launch_gemm(t, s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sa
