// Internal (host-side) interface between the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sa_sketch.h"

namespace sa {

struct WsHeader;

// ---- schedule: validates offsets, clears the status word, tile prefix sums
cudaError_t launch_schedule(const int64_t* offsets, int R, int64_t n_total, WsHeader* hdr,
                            long long* tile_start, cudaStream_t s);

// ---- fold: Pf[j][c] = scale * sum_e P[j][e] Wk[c][e] for j < k, 0 for k <= j < k_pad
cudaError_t launch_fold(const void* P, const void* Wk, sa_dtype dt, int k, int k_pad, int d,
                        float scale, void* Pf, bool out_bf16, cudaStream_t s);

// ---- finalize: sums a user's segment partials in order, then sketch = (U Wv) / mass
struct FinalizeArgs {
  const WsHeader* hdr;
  const long long* tile_start;
  const float* part_u;  // [segments, k_pad, d]
  const float* part_m;  // [segments, k_pad, mass_lanes]
  const void* Wv;
  sa_dtype dt;
  int R, k, k_pad, d, G;
  int H = 0, share = 0;  // helper ranges and their share of the tiles (TileRanges)
  int mass_lanes;       // partial masses per prototype and segment, summed in order
  float* sketch;
  float* mass;
  float* xsketch;  // nullable
  // tensor-core finalize (bf16, k = k_pad): U / mass as a bf16 pair hi + lo, [R, k, d] each
  __nv_bfloat16* ubar_hi;
  __nv_bfloat16* ubar_lo;
};
cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t s);
// Segment sums -> xsketch, mass and U / mass as hi + lo bf16; sketch = (hi + lo) Wv on the
// tensor cores (two accumulated GEMM phases). Needs ubar_hi / ubar_lo and k == k_pad.
cudaError_t launch_finalize_tc(const FinalizeArgs& a, cudaStream_t s);

// ---- combine: sketch = (U Wv) / mass from already summed U [R, k, d] and mass [R, k]
cudaError_t launch_combine(const float* U, const float* mass, int R, int k, int d, const void* Wv,
                           sa_dtype dt, float* sketch, cudaStream_t s);

// ---- tcgen05 forward (bf16)
struct FwdSm100Args {
  const CUtensorMap* tmap_x;
  const CUtensorMap* tmap_p;
  const int64_t* offsets;
  int R, k_valid, C, k_pad, d, G;
  int H = 0, share = 0;  // helper CTAs and their share of the tiles (TileRanges); 0: none
  WsHeader* hdr;
  const long long* tile_start;
  float* part_u;
  float* part_m;
  float* lse;
  long long budget;
};
cudaError_t fwd_sm100_max_clusters(int d, int C, int* n);
// Helper CTAs for the SMs that G clusters of C CTAs leave free, and their share of the
// tiles in 1/1024 (H = 0: none).
void fwd_sm100_helpers(int d, int C, int G, int sms, int* H, int* share);
// The clustered grid, then (a.H > 0) the helper grid, both on `stream`.
cudaError_t launch_fwd_sm100(const FwdSm100Args& a, cudaStream_t stream);
// The smallest workspace sa_sketch_forward accepts for these sizes (no helper grid); 0 if
// there is no plan.
size_t forward_workspace_min(int R, int64_t n_total, int k, int d, sa_dtype dt);

// ---- SIMT fp32 forward
struct FwdSimtArgs {
  const float* X;
  const int64_t* offsets;
  int R, k, k_pad, d, G;
  const float* Pf;  // folded prototypes [k_pad, d], log2 units
  WsHeader* hdr;
  const long long* tile_start;
  float* lse2;      // [n_total] workspace, log2 units
  float* lse;       // [n_total] user output (natural log), nullable
  int64_t n_total;
  float* part_u;
  float* part_m;
};
cudaError_t launch_fwd_simt(const FwdSimtArgs& a, cudaStream_t s);

// ---- SIMT backward
struct BwdArgs {
  const void* X;
  sa_dtype dt;
  const int64_t* offsets;
  int R, k, k_pad, d, G;
  int64_t n_total;
  const void* P;
  const void* Wk;
  const void* Wv;
  const float* sketch;
  const float* mass;
  const float* xsketch;
  const float* dsketch;
  const float* dmass;  // nullable
  WsHeader* hdr;
  const long long* tile_start;
  // workspace
  float* Pn;      // [k_pad, d]  P W_k^T / sqrt(d)
  float* Gt;      // [R, k_pad, d]  G / mass
  float* Gh;      // [R, k_pad, d]  (G / mass) W_v^T (nullable)
  __nv_bfloat16* Ghb;  // the same in bf16 (nullable; the tensor-core backward)
  __nv_bfloat16* Gtb;  // Gt in bf16 (nullable; the tensor-core backward)
  __nv_bfloat16* Gtlo; // bf16(Gt - bf16(Gt)) (nullable): Gh then comes from a tensor-core GEMM
  float* cj;      // [R, k_pad]     (G / mass) . sketch - dmass
  float* lseb;    // [n_total]      fp32 per-token log-sum-exp (natural)
  float* Db;      // [n_total]      sum_j A_jt dA_jt
  float* dpp_part;  // [G, k_pad, d]
  float* dpp;       // [k_pad, d]
  float* wv_part;   // [nchunks, d, d]
  // outputs
  float* dX;
  float* dP;
  float* dWk;
  float* dWv;
};
size_t bwd_wv_chunks(int R, int k);
cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_prep(const BwdArgs& a, cudaStream_t s);  // Gt, Gh, c per user
// dPn reduce, dW_v, dP, dW_k; wv_parts > 0: that many dW_v partials are already in wv_part
cudaError_t launch_bwd_tail(const BwdArgs& a, int wv_parts, cudaStream_t s);

// ---- single-pass backward kernel (sa_bwd_fused.cu)
struct BwdFusedArgs {
  const void* X;               // bf16 [n_total, d]
  const int64_t* offsets;
  int R, k_valid, C, k_pad, d, G;
  int64_t n_total;
  const WsHeader* hdr;
  const long long* tile_start;
  const __nv_bfloat16* pn;     // [k_pad, d] P W_k^T / sqrt(d)
  const __nv_bfloat16* gh;     // [R, k_pad, d] (G / mass) W_v^T
  const float* cj;             // [R, k_pad]
  const float* lse;            // [n_total] per-token log-sum-exp
  float lse_scale;             // lse2 = lse_scale * lse[t] (log2 units)
  float* dX;                   // [n_total, d], zeroed by the caller; partials are added
  float* dpp_part;             // [G, k_pad, d] per-cluster partials of dPn
  long long budget;
};
cudaError_t bwd_fused_max_clusters(int d, int C, int* n);
cudaError_t launch_bwd_fused(const BwdFusedArgs& a, cudaStream_t s);

// ---- tensor-core backward (bf16 inputs; sa_bwd_tc.cu)
struct BwdTcArgs {
  BwdArgs b;                 // shared inputs, outputs and SIMT-stage workspace
  const float* lse;          // forward's lse (natural log); null: recomputed here
  __nv_bfloat16* pn2;        // [k_pad, d] P W_k^T log2(e)/sqrt(d) (lse recompute only)
  __nv_bfloat16* pnn;        // [k_pad, d] P W_k^T / sqrt(d)
  float* dpart;              // [n_total, k_pad / 64] per-tile partials (lse recompute)
  float* lse2;               // [n_total] (when lse is null)
  __nv_bfloat16* Ub;         // [R, k_pad, d] bf16 xsketch (zero rows past k)
  int C, G;                  // cluster size and co-resident clusters of the fused kernel
  int wv_splits;             // split-K of dW_v (partials in b.wv_part)
};
cudaError_t launch_bwd_tc(const BwdTcArgs& a, cudaStream_t s);
int bwd_tc_wv_splits(int sms, int R, int k_pad);

// ---- tensor-core GEMM (backward building block, sa_gemm_sm100.cu)
enum GemmEpi { kEpiStoreF32 = 0, kEpiLse = 3, kEpiStoreBf16 = 4 };
struct GemmOperandDesc {  // one bf16 operand, row-major in memory
  const void* base;
  uint64_t rows, cols;
  bool mn_major;  // false: rows = M (or N), cols = K; true: rows = K, cols = M (or N)
};
struct GemmArgs {
  GemmOperandDesc a[2], b[2];  // operand pairs, accumulated into one result
  int phases;                  // 1 or 2
  int k_tiles[2];              // 64-wide K tiles of each pair
  int M, N;                    // rows and output columns
  int m_tiles_bound;           // grid x: 128-row tiles of M
  int splits;                  // split-K over pair 0's K tiles (grid z)
  int epi;
  const WsHeader* hdr;         // status word
  float* out_f32;
  long long ld_out;
  long long split_stride;
  __nv_bfloat16* out_bf16;
  int k_valid;                 // kEpiLse: columns n >= k_valid are padding
  float* dpart;
  int dpart_ld;
};
cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s);

// ---- candidate-to-sketch cross attention (sa_stca.cu)
struct StcaPlan {  // workspace layout (byte offsets, 256-aligned): the ragged-key
                   // attention's workspace first (its header is the status word), then the
                   // bf16 sketch, every user's row range within it and (backward) dKx
  int k_pad = 0;
  size_t hdr = 0, sb = 0, kb = 0, ke = 0, dkx = 0, total = 0;
};
size_t stca_plan(int R, long long n_cand, int k, int d, bool backward, int sms, StcaPlan* p);
struct StcaArgs {
  const void* Q;         // bf16 [n_cand, d]
  const int64_t* coff;   // [R + 1]
  int R, k, d;
  long long n_cand;
  const float* S;        // [R, k, d]
  const void* Wq;        // bf16 [d, d]
  const void* WK;
  const void* WV;
  float* out;            // [n_cand, d]
  float* lse;            // [n_cand] natural log, nullable
  void* workspace;
  StcaPlan plan;
};
cudaError_t launch_stca_forward(const StcaArgs& a, cudaStream_t s);
struct StcaGrads {
  const float* dout;          // [n_cand, d]
  float* dQ;                  // [n_cand, d]
  float* dS;                  // [R, k, d]
  float *dWq, *dWK, *dWV;     // [d, d]
};
cudaError_t launch_stca_backward(const StcaArgs& a, const StcaGrads& g, int sms, cudaStream_t s);

// shared pieces of the cross attention (sa_stca.cu)
cudaError_t stca_split_hilo(const float* x, long long n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                            cudaStream_t s);
cudaError_t stca_to_bf16(const float* x, long long n, __nv_bfloat16* y, cudaStream_t s);
cudaError_t stca_weight_grads(const float* dM, const void* Wq, const void* WK, int d, float* dWq,
                              float* dWK, cudaStream_t s);
cudaError_t gemm_hilo(const WsHeader* hdr, const __nv_bfloat16* hi, const __nv_bfloat16* lo,
                      long long n, int d, GemmOperandDesc bop, float* out, cudaStream_t s);
cudaError_t gemm_tn_sum(const WsHeader* hdr, const __nv_bfloat16* A, const __nv_bfloat16* B,
                        long long n, int d, int splits, float* part, float scale, float* out,
                        cudaStream_t s);

// ---- cross attention over ragged key rows (sa_stca_keys.cu)
struct StcaKeysPlan {  // workspace layout (byte offsets, 256-aligned)
  int splits = 0;
  size_t hdr = 0, ts = 0, mt = 0, qh = 0, ql = 0, o = 0, lse2 = 0, ohi = 0, olo = 0, total = 0;
  // backward only
  size_t mts = 0, ghi = 0, glo = 0, gb = 0, do_f = 0, do_b = 0, ob = 0, dd = 0, g1 = 0,
         g1hi = 0, g1lo = 0, part = 0, dm = 0;
};
size_t stca_keys_plan(int R, long long n_cand, int d, bool backward, int sms, StcaKeysPlan* p);
struct StcaKeysArgs {
  const void* Q;          // bf16 [n_cand, d]
  const int64_t* coff;    // [R + 1]
  int R, d;
  long long n_cand;
  const void* Kx;         // bf16 [n_keys, d]
  long long n_keys;
  const int64_t* kb;      // [R] first key row of each user
  const int64_t* ke;      // [R] one past its last key row
  const void* Wq;         // bf16 [d, d]
  const void* WK;
  const void* WV;
  float* out;             // [n_cand, d]
  float* lse;             // [n_cand] natural log, nullable
  void* workspace;
  StcaKeysPlan plan;
};
struct StcaKeysGrads {
  const float* dout;      // [n_cand, d]
  float* dQ;              // [n_cand, d]
  float* dKx;             // [n_keys, d]
  bool accumulate;        // add into dKx instead of overwriting it
  float *dWq, *dWK, *dWV; // [d, d]
};
cudaError_t launch_stca_keys_forward(const StcaKeysArgs& a, cudaStream_t s);
cudaError_t launch_stca_keys_backward(const StcaKeysArgs& a, const StcaKeysGrads& g,
                                      cudaStream_t s);
// the backward's tcgen05 kernel (sa_stca_keys_bwd.cu): G1 = sum_j dz_cj Kx_j per candidate
// (written) and dKx += ln 2 (dz^T Q' + (a log2 e)^T dO') per key row (added)
struct StcaKeysBwdArgs {
  const __nv_bfloat16* Qh;   // [n_cand, d] Q' hi
  const __nv_bfloat16* Ql;   // [n_cand, d] Q' lo
  const __nv_bfloat16* dOb;  // [n_cand, d] dL/dO' in bf16
  const void* Kx;            // bf16 [n_keys, d]
  long long n_keys, n_cand;
  const int64_t* coff;
  const int64_t* kb;
  const int64_t* ke;
  int R, d;
  const WsHeader* hdr;
  const long long* tile_start;  // the forward's candidate-tile schedule
  const float* lse2;         // [n_cand] log2 units
  const float* Dd;           // [n_cand] dO'_c . O'_c
  float* G1;                 // [n_cand, d] written
  float* dKx;                // [n_keys, d] added to (zeroed by the caller)
};
cudaError_t launch_stca_keys_bwd_kernel(const StcaKeysBwdArgs& a, cudaStream_t s);
// 2-D tensor map over bf16 rows [rows, cols]: boxes of 64 columns x 128 rows, 128B swizzle
bool tmap_rows_bf16(CUtensorMap* m, const void* base, uint64_t rows, int cols);
// key range of every user = its last min(n_u, L) history rows
cudaError_t launch_recent_ranges(const int64_t* offsets, int R, int64_t L, int64_t* kb,
                                 int64_t* ke, cudaStream_t s);

// ---- sketch cache codec (sa_codec.cu): format 0 = bf16, 1 = fp8 E4M3 with row scales
cudaError_t launch_sketch_pack(const float* S, long long rows, int d, int format, void* codes,
                               float* scales, cudaStream_t s);
cudaError_t launch_sketch_unpack(const void* codes, const float* scales, long long rows, int d,
                                 int format, float* S, cudaStream_t s);

// the measurement hook's events (sa_sketch_profile_events) recorded around a main kernel
extern thread_local cudaEvent_t g_prof_start;
extern thread_local cudaEvent_t g_prof_stop;
cudaError_t prof_mark_start(cudaStream_t s);
cudaError_t prof_mark_stop(cudaStream_t s);

// cuTensorMapEncodeTiled through the runtime's driver entry point (null if unavailable)
PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn();

// ---- failure-detection test hook
cudaError_t launch_debug_wait_timeout(WsHeader* hdr, long long budget, cudaStream_t s);

}  // namespace sa
