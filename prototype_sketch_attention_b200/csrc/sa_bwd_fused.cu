// Sketch Attention backward in one pass over the tokens (tcgen05, sm_100a), bf16 in /
// fp32 accumulate.
//
// The compression is differentiable (blog "100,000 videos in your pocket", section
// "1. Sketch Attention compresses the history"). With Pn = P W_k^T / sqrt(d), the
// forward's per-token log-sum-exp (lse2 in log2 units), and per user u
//   Gt = G / mass,  Gh = Gt W_v^T,  c_j = Gt_j . sketch_j - Gm_j   (the prep kernels)
// every token t of user u contributes
//   A_jt  = 2^(log2(e) Pn_j . X_t - lse2_t)
//   dA_jt = Gh_j . X_t - c_j
//   D_t   = sum_j A_jt dA_jt,   dS_jt = A_jt (dA_jt - D_t)
//   dX_t  = sum_j dS_jt Pn_j + sum_j A_jt Gh_j,   dPn += dS_t^T X_t.
//
// Decomposition: the forward's. A cluster of C = k_pad / 128 CTAs walks a contiguous
// range of 128-token tiles (a tile never spans users); CTA c owns prototypes
// [128c, 128c + 128). Per tile each CTA
//   1. loads X (TMA, 128B swizzle); Pn's slice is loaded once, Gh's slice and c's slice
//      whenever the tile's user changes;
//   2. tcgen05: S^T = X Pn_slice^T and dA'^T = X Gh_slice^T into TMEM (token = TMEM lane);
//   3. one thread per token: A = 2^(S log2 e - lse2), dA = dA' - c, the slice's part of
//      D_t, A as bf16 into shared memory; the partial D_t goes to every CTA of the
//      cluster (st.async into DSMEM) and comes back summed; then dS = A (dA - D) as bf16;
//   4. tcgen05: dX_part = dS Pn_slice + A Gh_slice (K = the slice's prototypes) into
//      TMEM, and dPn_slice += dS^T X, which accumulates in TMEM over the whole range;
//   5. an epilogue warpgroup moves dX_part out of TMEM through shared memory and adds it
//      into dX in global memory with TMA bulk reductions (cp.reduce.async.bulk.tensor
//      .add.f32, performed in L2): the C slices' partials of a token meet there. dX is
//      zeroed before the kernel. The order of those fp32 additions is not fixed, so dX
//      is not bitwise reproducible from run to run (dP, dW_k and dW_v are).
//   6. at the end of the range, dPn_slice goes to the workspace as this cluster's
//      partial; the tail kernel sums the clusters' partials in a fixed order.
// No token x prototype array touches HBM: per token the kernel reads X once and adds
// the C partial rows of dX.
//
// Roles: warp 0 TMA producer, warp 1 TMEM allocation and every MMA (in order), warps
// 4-7 the elementwise warpgroup, warps 8-11 the dX epilogue. Every mbarrier wait is
// bounded (see sa_common.cuh).
#include <cuda.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kSlice = 128;             // prototypes per CTA
constexpr int kBoxB = 16384;            // 128 rows x 128 bytes (64 bf16), 128B swizzle
constexpr int kStg = 128 * 16 * 4;      // dX staging chunk: 128 tokens x 16 fp32 (no swizzle)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColG = 128, kColX = 256, kColP = 384;
constexpr int kNS = 2;                  // X stages
constexpr int kThreads = 384;

// Shared memory (every MMA operand block 1024-byte aligned):
//   X stages   kNS x (d/64) boxes: X tile (K-major for the S and dA' MMAs, MN-major for
//              dPn += dS^T X)
//   Pn, Gh     (d/64) boxes each: K-major B of the S / dA' MMAs, MN-major B of dX_part
//   A, dS      two 16 KB blocks each (prototypes [0,64) and [64,128)), row = token:
//              K-major A of dX_part (M = tokens), and dS as the MN-major A of dPn
//   staging    2 x 8 KB fp32 blocks for the dX reductions
//   c          128 floats of the current user's c_j
//   exchange   NX slots x C x 128 floats (runtime C), then the barriers
template <int D, int NX>
struct BwdSmem {
  static constexpr int kXBoxes = D / 64;
  static constexpr int kXTile = kXBoxes * kBoxB;
  static constexpr int oX = 0;
  static constexpr int oPn = oX + kNS * kXTile;
  static constexpr int oGh = oPn + kXTile;
  static constexpr int oA = oGh + kXTile;
  static constexpr int oDS = oA + 2 * kBoxB;
  static constexpr int oStg = oDS + 2 * kBoxB;
  static constexpr int oC = oStg + 2 * kStg;
  static constexpr int oXch = oC + kSlice * 4;
  __host__ __device__ static constexpr int xbox(int s, int b) { return oX + s * kXTile + b * kBoxB; }
  __host__ __device__ static size_t bars_off(int C) { return (size_t)oXch + (size_t)NX * C * 512; }
};

struct BwdBars {
  uint64_t x_full[kNS], x_empty[kNS];
  uint64_t p_full, g_full, g_empty;
  uint64_t s_full, ds_full;
  uint64_t dx_full, dx_empty, dp_full;
  uint64_t stg_full[2], stg_free[2];
  uint64_t xch[4];
  uint64_t drain;
  uint32_t tmem_base;
};

template <int D, int NX>
size_t smem_bytes_t(int C) {
  return 1024 + BwdSmem<D, NX>::bars_off(C) + sizeof(BwdBars);
}

// 1-D bulk copy global -> this CTA's shared memory, completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// 2-D TMA reduction: global tile at (x, y) += the shared-memory box, fp32 add in L2.
__device__ __forceinline__ void tma_reduce_add_2d(const void* tmap, int x, int y, uint32_t src) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];"
      ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One 32-prototype half block (4 chunks of 16 bytes starting at chunk ch0) of token row r
// into a 128B-swizzled [token][64 prototypes] block.
__device__ __forceinline__ void store_half(uint8_t* rowp, int r, int ch0, const uint32_t (&pk)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(rowp + (((ch0 + j) ^ (r & 7)) << 4)) =
        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
}
__device__ __forceinline__ void load_half(const uint8_t* rowp, int r, int ch0, uint32_t (&pk)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 v = *reinterpret_cast<const uint4*>(rowp + (((ch0 + j) ^ (r & 7)) << 4));
    pk[4 * j] = v.x;
    pk[4 * j + 1] = v.y;
    pk[4 * j + 2] = v.z;
    pk[4 * j + 3] = v.w;
  }
}

template <int D, int NX>
__global__ void __launch_bounds__(kThreads, 1)
sa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_pn,
                    const __grid_constant__ CUtensorMap tmap_gh,
                    const __grid_constant__ CUtensorMap tmap_dx,
                    const int64_t* __restrict__ offsets, int R, int k_valid, int C, int k_pad,
                    const WsHeader* hdr_c, const long long* __restrict__ tile_start,
                    const float* __restrict__ lse, float lse_scale, const float* __restrict__ cj,
                    float* __restrict__ dpp_part, long long budget) {
  using L = BwdSmem<D, NX>;
  constexpr int KS_D = D / 16;        // K steps over d
  constexpr int KS_T = 128 / 16;      // K steps over 128 prototypes or 128 tokens
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* xch = reinterpret_cast<float*>(smem + L::oXch);
  const float* csm = reinterpret_cast<const float*>(smem + L::oC);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + L::bars_off(C));
  WsHeader* hdr = const_cast<WsHeader*>(hdr_c);
  int* status = &hdr->status;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t cid = cluster_id_x(), ncl = nclusters_x();
  const int pbase = (int)rank * kSlice;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(smem_u32(&bars->x_full[s]), 1);
      mbar_init(smem_u32(&bars->x_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->p_full), 1);
    mbar_init(smem_u32(&bars->g_full), 1);
    mbar_init(smem_u32(&bars->g_empty), 1);
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->ds_full), 4);
    mbar_init(smem_u32(&bars->dx_full), 1);
    mbar_init(smem_u32(&bars->dx_empty), 4);
    mbar_init(smem_u32(&bars->dp_full), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->stg_full[b]), 4);
      mbar_init(smem_u32(&bars->stg_free[b]), 1);
    }
    for (int q = 0; q < NX; ++q) mbar_init(smem_u32(&bars->xch[q]), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // peers' barriers are initialised before any st.async arrives
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const long long T = read_status(status) == 0 ? hdr->total_tiles : 0;
  const long long ta = (long long)cid * T / ncl, tb = (long long)(cid + 1) * T / ncl;

  if (warp == 0) {
    // ================= TMA producer: Pn once; per segment Gh and c; X per tile
    if (lane == 0 && ta < tb) {
      tma_prefetch_desc(&tmap_x);
      tma_prefetch_desc(&tmap_pn);
      tma_prefetch_desc(&tmap_gh);
      const uint32_t pf = smem_u32(&bars->p_full);
      mbar_arrive_expect_tx(pf, L::kXTile);
      for (int b = 0; b < L::kXBoxes; ++b)
        tma_load_2d(sbase + L::oPn + b * kBoxB, &tmap_pn, b * 64, pbase, pf);
      TileIter it;
      it.init(tile_start, offsets, R, ta, tb);
      int i = 0, seg = -1, prev_u = -1;
      bool ok = true;
      for (; ok && it.valid(); it.next(), ++i) {
        if (it.u != prev_u) {  // a new segment: Gh and c of user it.u
          prev_u = it.u;
          ++seg;
          if (!mbar_wait(smem_u32(&bars->g_empty), (uint32_t)((seg & 1) ^ 1), status, budget)) break;
          const uint32_t gf = smem_u32(&bars->g_full);
          mbar_arrive_expect_tx(gf, L::kXTile + kSlice * 4);
          for (int b = 0; b < L::kXBoxes; ++b)
            tma_load_2d(sbase + L::oGh + b * kBoxB, &tmap_gh, b * 64, it.u * k_pad + pbase, gf);
          bulk_load(sbase + L::oC, cj + (size_t)it.u * k_pad + pbase, kSlice * 4, gf);
        }
        const int st = i % kNS;
        if (!mbar_wait(smem_u32(&bars->x_empty[st]), (uint32_t)(((i / kNS) & 1) ^ 1), status, budget))
          break;
        const uint32_t fb = smem_u32(&bars->x_full[st]);
        mbar_arrive_expect_tx(fb, L::kXTile);
        for (int b = 0; b < L::kXBoxes; ++b)
          tma_load_2d(sbase + L::xbox(st, b), &tmap_x, b * 64, (int)it.t0(), fb);
      }
      // drain: every load issued must have landed before exit
      for (int j = (i > kNS ? i - kNS : 0); j < i; ++j)
        mbar_wait_drain(smem_u32(&bars->x_full[j % kNS]), (uint32_t)((j / kNS) & 1), budget);
      if (seg >= 0) mbar_wait_drain(smem_u32(&bars->g_full), (uint32_t)(seg & 1), budget);
      mbar_wait_drain(pf, 0, budget);
    }
  } else if (warp == 1) {
    // ================= MMA issuer: per tile S, dA' then (after the elementwise pass)
    // dX_part and dPn, all in issue order on one tensor pipe
    if (lane == 0 && ta < tb) {
      const uint32_t id_sg = idesc_bf16_f32(128, kSlice, 0, 0);   // X (K) x Pn / Gh (K)
      const uint32_t id_dx = idesc_bf16_f32(128, D, 0, 1);        // dS / A (K) x Pn / Gh (MN)
      const uint32_t id_dp = idesc_bf16_f32(128, D, 1, 1);        // dS^T (MN) x X (MN)
      const uint64_t d_pn_k = smem_desc(sbase + L::oPn, 16, 1024, kSwizzle128B);
      const uint64_t d_gh_k = smem_desc(sbase + L::oGh, 16, 1024, kSwizzle128B);
      const uint64_t d_pn_mn = smem_desc(sbase + L::oPn, kBoxB, 1024, kSwizzle128B);
      const uint64_t d_gh_mn = smem_desc(sbase + L::oGh, kBoxB, 1024, kSwizzle128B);
      const uint64_t d_ds_k = smem_desc(sbase + L::oDS, 16, 1024, kSwizzle128B);
      const uint64_t d_a_k = smem_desc(sbase + L::oA, 16, 1024, kSwizzle128B);
      const uint64_t d_ds_mn = smem_desc(sbase + L::oDS, kBoxB, 1024, kSwizzle128B);
      bool ok = mbar_wait(smem_u32(&bars->p_full), 0, status, budget);
      TileIter it;
      it.init(tile_start, offsets, R, ta, tb);
      int i = 0, seg = -1, prev_u = -1;
      for (; ok && it.valid(); it.next(), ++i) {
        const bool first = it.u != prev_u, last = it.last();
        prev_u = it.u;
        if (first) ++seg;
        const int st = i % kNS;
        ok = mbar_wait(smem_u32(&bars->x_full[st]), (uint32_t)((i / kNS) & 1), status, budget) &&
             (!first || mbar_wait(smem_u32(&bars->g_full), (uint32_t)(seg & 1), status, budget));
        if (!ok) break;
        tc_fence_after();
        // S^T and dA'^T: A = X tile (K-major, four 16-wide K steps per 64-column box)
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
          const uint64_t xa = smem_desc(sbase + L::xbox(st, ks >> 2), 16, 1024, kSwizzle128B) +
                              (uint64_t)(((ks & 3) * 32) >> 4);
          const uint64_t koff = (uint64_t)((((ks >> 2) * kBoxB) + (ks & 3) * 32) >> 4);
          tc_mma_f16(tmem + kColS, xa, d_pn_k + koff, id_sg, ks > 0 ? 1u : 0u);
          tc_mma_f16(tmem + kColG, xa, d_gh_k + koff, id_sg, ks > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&bars->s_full));
        // the elementwise pass has stored A and dS and read S and dA' (ds_full), and the
        // epilogue has taken dX_part of the previous tile out of TMEM (dx_empty)
        ok = mbar_wait(smem_u32(&bars->ds_full), (uint32_t)(i & 1), status, budget) &&
             mbar_wait(smem_u32(&bars->dx_empty), (uint32_t)((i & 1) ^ 1), status, budget);
        if (!ok) break;
        tc_fence_after();
        // dX_part = dS Pn_slice + A Gh_slice: K = the slice's 128 prototypes; the K-major
        // A operand advances 32 bytes per step within a 64-prototype block, the MN-major B
        // operand two 8-row groups (2048 bytes) per step
#pragma unroll
        for (int ks = 0; ks < KS_T; ++ks) {
          const uint64_t ka = (uint64_t)((((ks >> 2) * kBoxB) + (ks & 3) * 32) >> 4);
          const uint64_t kb = (uint64_t)((ks * 2048) >> 4);
          tc_mma_f16(tmem + kColX, d_ds_k + ka, d_pn_mn + kb, id_dx, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < KS_T; ++ks) {
          const uint64_t ka = (uint64_t)((((ks >> 2) * kBoxB) + (ks & 3) * 32) >> 4);
          const uint64_t kb = (uint64_t)((ks * 2048) >> 4);
          tc_mma_f16(tmem + kColX, d_a_k + ka, d_gh_mn + kb, id_dx, 1u);
        }
        tc_commit(smem_u32(&bars->dx_full));
        // dPn_slice += dS^T X: A = dS (MN-major, M = prototypes), B = X (MN-major, N = d)
        const uint64_t d_x_mn = smem_desc(sbase + L::xbox(st, 0), kBoxB, 1024, kSwizzle128B);
#pragma unroll
        for (int ks = 0; ks < KS_T; ++ks)
          tc_mma_f16(tmem + kColP, d_ds_mn + (uint64_t)((ks * 2048) >> 4),
                     d_x_mn + (uint64_t)((ks * 2048) >> 4), id_dp, (i == 0 && ks == 0) ? 0u : 1u);
        tc_commit(smem_u32(&bars->x_empty[st]));
        if (last) tc_commit(smem_u32(&bars->g_empty));
      }
      tc_commit(smem_u32(&bars->dp_full));
      tc_commit(smem_u32(&bars->drain));
      mbar_wait_drain(smem_u32(&bars->drain), 0, budget);
    }
  } else if (warp >= 4 && warp < 8) {
    // ================= elementwise warpgroup: thread = token row = TMEM lane
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const bool leader = threadIdx.x == 128;
    const int ncols = min(kSlice, k_valid - pbase);
    uint8_t* arow[2] = {smem + L::oA + r * 128, smem + L::oA + kBoxB + r * 128};
    uint8_t* drow[2] = {smem + L::oDS + r * 128, smem + L::oDS + kBoxB + r * 128};
    TileIter it;
    it.init(tile_start, offsets, R, ta, tb);
    int i = 0, seg = -1, prev_u = -1;
    bool ok = true;
    for (; ok && it.valid(); it.next(), ++i) {
      const bool first = it.u != prev_u;
      prev_u = it.u;
      if (first) ++seg;
      const bool valid = r < it.nvalid();
      const float l2 = valid ? lse[it.t0() + r] * lse_scale : 0.f;
      if (!mbar_wait_warp(smem_u32(&bars->s_full), (uint32_t)(i & 1), status, budget) ||
          (first && !mbar_wait_warp(smem_u32(&bars->g_full), (uint32_t)(seg & 1), status, budget))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 1: A = 2^(S log2 e - lse2) (bf16 into the A tile), the slice's part of D
      float dsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t s32[32], g32[32], pk[16];
        tmem_ld32_raw(tmem + lane_off + kColS + c * 32, s32);
        tmem_ld32_raw(tmem + lane_off + kColG + c * 32, g32);
        tmem_wait_tie(s32);
        tmem_wait_tie(g32);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const int j = c * 32 + 2 * p;
          float a0 = 0.f, a1 = 0.f;
          if (valid && j < ncols) a0 = ex2_approx(fmaf(__uint_as_float(s32[2 * p]), 1.4426950408889634f, -l2));
          if (valid && j + 1 < ncols) a1 = ex2_approx(fmaf(__uint_as_float(s32[2 * p + 1]), 1.4426950408889634f, -l2));
          dsum = fmaf(a0, __uint_as_float(g32[2 * p]) - csm[j], dsum);
          dsum = fmaf(a1, __uint_as_float(g32[2 * p + 1]) - csm[j + 1], dsum);
          pk[p] = cvt_bf16x2(a0, a1);
        }
        store_half(arow[c >> 1], r, (c & 1) * 4, pk);
      }
      // exchange the partial D_t with every CTA of the cluster (4 tokens per st.async)
      const int qs = i % NX;
      const uint32_t xbar = smem_u32(&bars->xch[qs]);
      {
        const int g0 = lane & ~3;
        const float v0 = __shfl_sync(0xffffffffu, dsum, g0 + 0);
        const float v1 = __shfl_sync(0xffffffffu, dsum, g0 + 1);
        const float v2 = __shfl_sync(0xffffffffu, dsum, g0 + 2);
        const float v3 = __shfl_sync(0xffffffffu, dsum, g0 + 3);
        const uint32_t laddr = smem_u32(xch + ((qs * C + (int)rank) * 128 + q4 * 32 + g0));
        for (int p = lane & 3; p < C; p += 4)
          st_async_v4(mapa(laddr, (uint32_t)p), v0, v1, v2, v3, mapa(xbar, (uint32_t)p));
      }
      if (leader) mbar_arrive_expect_tx(xbar, (uint32_t)C * 512u);
      if (!mbar_wait_warp<true>(xbar, (uint32_t)((i / NX) & 1), status, budget)) {
        ok = false;
        break;
      }
      float Dt = 0.f;
      for (int p = 0; p < C; ++p) Dt += xch[(qs * C + p) * 128 + r];  // fixed order
      // pass 2: dS = A (dA' - c - D) as bf16 into the dS tile
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t g32[32], ak[16], pk[16];
        tmem_ld32_raw(tmem + lane_off + kColG + c * 32, g32);
        load_half(arow[c >> 1], r, (c & 1) * 4, ak);
        tmem_wait_tie(g32);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const int j = c * 32 + 2 * p;
          const float a0 = __uint_as_float(ak[p] << 16), a1 = __uint_as_float(ak[p] & 0xFFFF0000u);
          const float d0 = a0 * (__uint_as_float(g32[2 * p]) - csm[j] - Dt);
          const float d1 = a1 * (__uint_as_float(g32[2 * p + 1]) - csm[j + 1] - Dt);
          pk[p] = cvt_bf16x2(d0, d1);
        }
        store_half(drow[c >> 1], r, (c & 1) * 4, pk);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full));
    }
  } else if (warp >= 8) {
    // ================= dX epilogue: TMEM -> shared staging -> TMA reduce-add into dX
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const bool issuer = threadIdx.x == 256;
    constexpr int kChunks = D / 16;
    TileIter it;
    it.init(tile_start, offsets, R, ta, tb);
    int i = 0, n = 0;  // n: staging chunks used so far (buffer n & 1, phase n >> 1)
    bool ok = true;
    for (; ok && it.valid(); it.next(), ++i) {
      if (!mbar_wait_warp(smem_u32(&bars->dx_full), (uint32_t)(i & 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int y = (int)it.t0();
      for (int h = 0; h < D / 32; ++h) {
        uint32_t v[32];
        tmem_ld32_raw(tmem + lane_off + kColX + h * 32, v);
        tmem_wait_tie(v);
        if (h == D / 32 - 1) {  // dX_part fully in registers: TMEM is free for the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->dx_empty));
        }
#pragma unroll
        for (int half = 0; half < 2; ++half, ++n) {
          const int b = n & 1;
          // this buffer's previous reduction has finished reading it
          if (n >= 2 && !mbar_wait_warp(smem_u32(&bars->stg_free[b]), (uint32_t)(((n >> 1) - 1) & 1),
                                        status, budget)) {
            ok = false;
            break;
          }
          float4* dst = reinterpret_cast<float4*>(smem + L::oStg + b * kStg + r * 64);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_float4(__uint_as_float(v[half * 16 + 4 * x]), __uint_as_float(v[half * 16 + 4 * x + 1]),
                                 __uint_as_float(v[half * 16 + 4 * x + 2]),
                                 __uint_as_float(v[half * 16 + 4 * x + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->stg_full[b]));
          if (issuer) {
            if (!mbar_wait(smem_u32(&bars->stg_full[b]), (uint32_t)((n >> 1) & 1), status, budget)) {
              ok = false;
            } else {
              tma_reduce_add_2d(&tmap_dx, (h * 2 + half) * 16, y, sbase + L::oStg + b * kStg);
              bulk_commit();
              bulk_wait_read<0>();
              mbar_arrive(smem_u32(&bars->stg_free[b]));
            }
          }
        }
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
      }
      (void)kChunks;
    }
    if (issuer) bulk_wait_all();
    // ---- this cluster's dPn_slice partial (TMEM lane = prototype), zeros if it had no tiles
    float* dst = dpp_part + ((size_t)cid * k_pad + pbase + r) * D;
    const bool have = ok && ta < tb && mbar_wait_warp(smem_u32(&bars->dp_full), 0, status, budget);
    if (have) tc_fence_after();
#pragma unroll
    for (int h = 0; h < D / 32; ++h) {
      uint32_t v[32];
      if (have) {
        tmem_ld32_raw(tmem + lane_off + kColP + h * 32, v);
        tmem_wait_tie(v);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = 0u;
      }
#pragma unroll
      for (int x = 0; x < 32; x += 4)
        *reinterpret_cast<float4*>(dst + h * 32 + x) =
            make_float4(__uint_as_float(v[x]), __uint_as_float(v[x + 1]), __uint_as_float(v[x + 2]),
                        __uint_as_float(v[x + 3]));
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no peer touches our shared memory after this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int NX>
cudaError_t configure_t(int C, size_t* smem) {
  auto kern = sa_bwd_fused_kernel<D, NX>;
  *smem = smem_bytes_t<D, NX>(C);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)*smem);
  if (e != cudaSuccess) return e;
  if (C > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int D, int NX>
cudaError_t max_clusters_t(int C, int* n) {
  size_t smem = 0;
  cudaError_t e = configure_t<D, NX>(C, &smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(n, sa_bwd_fused_kernel<D, NX>, &cfg);
}

// Row-major [rows, cols] tensor maps: bf16 operands in 64-column boxes of 128 rows with
// the 128-byte swizzle; the fp32 dX in 16-column boxes of 128 rows, unswizzled.
bool map_bf16(CUtensorMap* m, const void* base, uint64_t rows, int cols) {
  auto fn = tmap_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool map_f32_rows(CUtensorMap* m, void* base, uint64_t rows, int cols) {
  auto fn = tmap_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  const cuuint32_t box[2] = {16, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NX>
cudaError_t launch_t(const BwdFusedArgs& a, cudaStream_t s) {
  CUtensorMap tx, tpn, tgh, tdx;
  if (!map_bf16(&tx, a.X, (uint64_t)a.n_total, a.d) || !map_bf16(&tpn, a.pn, (uint64_t)a.k_pad, a.d) ||
      !map_bf16(&tgh, a.gh, (uint64_t)a.R * a.k_pad, a.d) ||
      !map_f32_rows(&tdx, a.dX, (uint64_t)a.n_total, a.d))
    return cudaErrorInvalidValue;
  size_t smem = 0;
  cudaError_t e = configure_t<D, NX>(a.C, &smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.G * a.C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sa_bwd_fused_kernel<D, NX>, tx, tpn, tgh, tdx, a.offsets, a.R,
                            a.k_valid, a.C, a.k_pad, a.hdr, a.tile_start, a.lse, a.lse_scale, a.cj,
                            a.dpp_part, a.budget);
}

}  // namespace

// Exchange slots: 2 (the single elementwise warpgroup handles tiles in order, so a slot
// is read before any CTA can send the tile two ahead into it).
cudaError_t bwd_fused_max_clusters(int d, int C, int* n) {
  return d == 64 ? max_clusters_t<64, 2>(C, n) : max_clusters_t<128, 2>(C, n);
}

cudaError_t launch_bwd_fused(const BwdFusedArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_t<64, 2>(a, s) : launch_t<128, 2>(a, s);
}

}  // namespace sa
