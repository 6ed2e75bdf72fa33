// Candidate-to-sketch cross attention (the sketch branch of STCA) on the tensor cores.
//
// User u has a sketch S_u [k, d] (Sketch Attention's output) and candidates Q_c,
// c in [coff[u], coff[u+1]); every candidate of the user reads that one sketch:
//   out_c = sum_j softmax_j( (Q_c W_q) . (S_uj W_K) / sqrt(d) ) S_uj W_V
// ("100,000 videos in your pocket" blog, sections "2. STCA reasons at two time scales",
// the sketch branch, and "3. The system makes it cheap enough to matter", multi-request
// user-level batching). This is the ragged-key cross attention of sa_stca_keys.cu with
// the sketch rows as the keys: the sketch goes to bf16 [R, k_pad, d] (rows past k zero),
// user u's key range is the rows [u k_pad, u k_pad + k), and both directions run that
// file's kernels. The backward's dKx over those rows is dS, the gradient that flows into
// each user's sketch (Sketch Attention's dL/dsketch); a last kernel drops the pad rows.
//
// The pieces that both cross attentions share live here too: bf16 conversions, the
// hi + lo split, the weight gradients and the GEMM compositions on the tcgen05 GEMM.
#include <cmath>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

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
  StcaKeysPlan kp;  // the ragged-key attention's workspace first: its header is the status word
  size_t o = stca_keys_plan(R, n_cand, d, backward, sms, &kp);
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 255) / 256 * 256;
    return at;
  };
  q.hdr = kp.hdr;
  q.sb = take((size_t)R * q.k_pad * d * 2);
  q.kb = take((size_t)R * sizeof(int64_t));
  q.ke = take((size_t)R * sizeof(int64_t));
  if (backward) q.dkx = take((size_t)R * q.k_pad * d * sizeof(float));
  q.total = o;
  *p = q;
  return o;
}

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

namespace {

// The sketch as the key rows: bf16 [R, k_pad, d] and every user's range within it.
cudaError_t sketch_keys(const StcaArgs& a, StcaKeysArgs* k, cudaStream_t s) {
  const StcaPlan& p = a.plan;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  __nv_bfloat16* Sb = reinterpret_cast<__nv_bfloat16*>(ws + p.sb);
  int64_t* kb = reinterpret_cast<int64_t*>(ws + p.kb);
  int64_t* ke = reinterpret_cast<int64_t*>(ws + p.ke);
  if (a.R > 0) {
    stca_sketch_bf16_kernel<<<1024, 256, 0, s>>>(a.S, a.R, a.k, p.k_pad, a.d, Sb);
    stca_sketch_ranges_kernel<<<(a.R + 255) / 256, 256, 0, s>>>(a.R, a.k, p.k_pad, kb, ke);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  k->Q = a.Q;
  k->coff = a.coff;
  k->R = a.R;
  k->d = a.d;
  k->n_cand = a.n_cand;
  k->Kx = Sb;
  k->n_keys = (long long)a.R * p.k_pad;
  k->kb = kb;
  k->ke = ke;
  k->Wq = a.Wq;
  k->WK = a.WK;
  k->WV = a.WV;
  k->out = a.out;
  k->lse = a.lse;
  k->workspace = a.workspace;
  return cudaSuccess;
}

// dS [R, k, d] = the rows [u k_pad, u k_pad + k) of dKx [R k_pad, d].
__global__ void stca_ds_rows_kernel(const float4* __restrict__ dkx, int R, int k, int k_pad, int d,
                                    float4* __restrict__ dS) {
  const int d4 = d / 4;
  const long long n = (long long)R * k * d4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i % d4, rj = i / d4, j = rj % k, u = rj / k;
    dS[i] = dkx[(u * k_pad + j) * d4 + e];
  }
}

}  // namespace

cudaError_t launch_stca_forward(const StcaArgs& a, cudaStream_t s) {
  StcaKeysArgs k;
  cudaError_t e = sketch_keys(a, &k, s);
  if (e != cudaSuccess) return e;
  stca_keys_plan(a.R, a.n_cand, a.d, false, 0, &k.plan);
  return launch_stca_keys_forward(k, s);
}

cudaError_t launch_stca_backward(const StcaArgs& a, const StcaGrads& gr, int sms, cudaStream_t s) {
  StcaKeysArgs k;
  cudaError_t e = sketch_keys(a, &k, s);
  if (e != cudaSuccess) return e;
  stca_keys_plan(a.R, a.n_cand, a.d, true, sms, &k.plan);
  StcaKeysGrads g;
  g.dout = gr.dout;
  g.dQ = gr.dQ;
  g.dKx = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + a.plan.dkx);
  g.accumulate = false;
  g.dWq = gr.dWq;
  g.dWK = gr.dWK;
  g.dWV = gr.dWV;
  if ((e = launch_stca_keys_backward(k, g, s)) != cudaSuccess) return e;
  if (a.R == 0) return cudaSuccess;
  stca_ds_rows_kernel<<<1024, 256, 0, s>>>(reinterpret_cast<const float4*>(g.dKx), a.R, a.k,
                                           a.plan.k_pad, a.d, reinterpret_cast<float4*>(gr.dS));
  return cudaGetLastError();
}

}  // namespace sa
