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
//   3. one thread per token and half slice: A = 2^(S log2 e - lse2) (written back into
//      TMEM as bf16 pairs over the S it replaces), dA = dA' - c, the slice's part of D_t;
//      the partial D_t goes to every CTA of the cluster (st.async into DSMEM) and comes
//      back summed; then dS = A (dA - D), and A and dS go to shared memory as bf16;
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
// Roles: warp 0 TMA producer, warp 1 TMEM allocation and every MMA (in order), warp 2
// the dX reductions, warps 4-11 two elementwise warpgroups (half of the slice's
// prototypes each), warps 12-15 the dX epilogue. Every mbarrier wait is bounded (see
// sa_common.cuh).
#include <cuda.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kSlice = 128;             // prototypes per CTA
constexpr int kBoxB = 16384;            // 128 rows x 128 bytes (64 bf16), 128B swizzle
constexpr int kStg = 128 * 16 * 4;      // dX staging chunk: 128 tokens x 16 fp32, 64B swizzle
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColG = 128, kColX = 256, kColP = 384;
constexpr int kNS = 2;                  // X stages
constexpr int kThreads = 512;

// Shared memory (every MMA operand block 1024-byte aligned):
//   X stages   kNS x (d/64) boxes: X tile (K-major for the S and dA' MMAs, MN-major for
//              dPn += dS^T X)
//   Pn, Gh     (d/64) boxes each: K-major B of the S / dA' MMAs, MN-major B of dX_part
//   A, dS      two 16 KB blocks each (prototypes [0,64) and [64,128)), row = token:
//              K-major A of dX_part (M = tokens), and dS as the MN-major A of dPn
//   staging    NB x 8 KB fp32 blocks for the dX reductions (64-byte rows, 64B swizzle)
//   c          128 floats of the current user's c_j
//   dhalf      128 floats: the second elementwise warpgroup's half of D_t
//   exchange   NX slots x C x 128 floats (runtime C), then the barriers
template <int D, int NX, int NB>
struct BwdSmem {
  static constexpr int kXBoxes = D / 64;
  static constexpr int kXTile = kXBoxes * kBoxB;
  static constexpr int oX = 0;
  static constexpr int oPn = oX + kNS * kXTile;
  static constexpr int oGh = oPn + kXTile;
  static constexpr int oA = oGh + kXTile;
  static constexpr int oDS = oA + 2 * kBoxB;
  static constexpr int oStg = oDS + 2 * kBoxB;
  static constexpr int oC = oStg + NB * kStg;
  static constexpr int oDh = oC + kSlice * 4;
  static constexpr int oXch = oDh + 128 * 4;
  __host__ __device__ static constexpr int xbox(int s, int b) { return oX + s * kXTile + b * kBoxB; }
  __host__ __device__ static size_t bars_off(int C) { return (size_t)oXch + (size_t)NX * C * 512; }
};

struct BwdBars {
  uint64_t x_full[kNS], x_empty[kNS];
  uint64_t p_full, g_full, g_empty;
  uint64_t sS_full, sG_full, ds_full, dhalf, tiles_free;
  uint64_t dx_full, dx_empty, dp_full;
  uint64_t stg_full[3], stg_free[3];
  uint64_t xch[4];
  uint64_t drain;
  uint32_t tmem_base;
};

template <int D, int NX, int NB>
size_t smem_bytes_t(int C) {
  return 1024 + BwdSmem<D, NX, NB>::bars_off(C) + sizeof(BwdBars);
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

// 32 lanes x 8 consecutive 32-bit TMEM columns from / into registers (thread i of the
// warp <-> lane base + i).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                 "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit TMEM columns into registers; the wait carries the
// registers so that no use is scheduled before it.
__device__ __forceinline__ void tmem_wait8(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7])
               :
               : "memory");
}

template <int D, int NX, int NB>
__global__ void __launch_bounds__(kThreads, 1)
sa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_pn,
                    const __grid_constant__ CUtensorMap tmap_gh,
                    const __grid_constant__ CUtensorMap tmap_dx,
                    const int64_t* __restrict__ offsets, int R, int k_valid, int C, int k_pad,
                    const WsHeader* hdr_c, const long long* __restrict__ tile_start,
                    const float* __restrict__ lse, float lse_scale, const float* __restrict__ cj,
                    float* __restrict__ dpp_part, long long budget) {
  using L = BwdSmem<D, NX, NB>;
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
    mbar_init(smem_u32(&bars->sS_full), 1);
    mbar_init(smem_u32(&bars->sG_full), 1);
    mbar_init(smem_u32(&bars->ds_full), 8);
    mbar_init(smem_u32(&bars->dhalf), 4);
    mbar_init(smem_u32(&bars->tiles_free), 1);
    mbar_init(smem_u32(&bars->dx_full), 1);
    mbar_init(smem_u32(&bars->dx_empty), 4);
    mbar_init(smem_u32(&bars->dp_full), 1);
    for (int b = 0; b < NB; ++b) {
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
    // ================= MMA issuer, all on one in-order tensor pipe. Per tile i: S(i) and
    // dA'(i); once the elementwise pass has stored A(i) and dS(i), S(i + 1) and dA'(i + 1)
    // go first when tile i + 1 belongs to the same user (its pass 1 then overlaps the
    // rest), then dX_part(i) and dPn += dS(i)^T X(i). At a user boundary the new user's
    // Gh replaces the old one only after dX_part(i) has read it, so S(i + 1) and
    // dA'(i + 1) follow.
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
      // S^T then dA'^T of tile j, each with its own commit (the exponentials need only S):
      // A = X tile (K-major, four 16-wide K steps per 64-column box)
      auto issue_sg = [&](int j) {
        const int st = j % kNS;
        uint64_t xa[KS_D];
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks)
          xa[ks] = smem_desc(sbase + L::xbox(st, ks >> 2), 16, 1024, kSwizzle128B) +
                   (uint64_t)(((ks & 3) * 32) >> 4);
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks)
          tc_mma_f16(tmem + kColS, xa[ks], d_pn_k + (uint64_t)((((ks >> 2) * kBoxB) + (ks & 3) * 32) >> 4),
                     id_sg, ks > 0 ? 1u : 0u);
        tc_commit(smem_u32(&bars->sS_full));
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks)
          tc_mma_f16(tmem + kColG, xa[ks], d_gh_k + (uint64_t)((((ks >> 2) * kBoxB) + (ks & 3) * 32) >> 4),
                     id_sg, ks > 0 ? 1u : 0u);
        tc_commit(smem_u32(&bars->sG_full));
      };
      bool ok = mbar_wait(smem_u32(&bars->p_full), 0, status, budget);
      TileIter it;
      it.init(tile_start, offsets, R, ta, tb);
      int i = 0, seg = 0;
      ok = ok && mbar_wait(smem_u32(&bars->x_full[0]), 0, status, budget) &&
           mbar_wait(smem_u32(&bars->g_full), 0, status, budget);
      if (ok) {
        tc_fence_after();
        issue_sg(0);
      }
      while (ok && it.valid()) {
        const int st = i % kNS;
        const bool last = it.last();  // last tile of its user (or of the range)
        it.next();
        const bool more = it.valid(), same = more && !last;
        const int s1 = (i + 1) % kNS;
        // the elementwise pass has stored A(i), dS(i) and read S(i), dA'(i)
        ok = mbar_wait(smem_u32(&bars->ds_full), (uint32_t)(i & 1), status, budget);
        if (!ok) break;
        if (same) {
          ok = mbar_wait(smem_u32(&bars->x_full[s1]), (uint32_t)(((i + 1) / kNS) & 1), status, budget);
          if (!ok) break;
          tc_fence_after();
          issue_sg(i + 1);
        }
        // the epilogue has taken dX_part(i - 1) out of TMEM
        ok = mbar_wait(smem_u32(&bars->dx_empty), (uint32_t)((i & 1) ^ 1), status, budget);
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
        tc_commit(smem_u32(&bars->tiles_free));
        if (last) tc_commit(smem_u32(&bars->g_empty));
        if (more && !same) {  // the next user's first tile, once its Gh has landed
          ++seg;
          ok = mbar_wait(smem_u32(&bars->x_full[s1]), (uint32_t)(((i + 1) / kNS) & 1), status, budget) &&
               mbar_wait(smem_u32(&bars->g_full), (uint32_t)(seg & 1), status, budget);
          if (!ok) break;
          tc_fence_after();
          issue_sg(i + 1);
        }
        ++i;
      }
      tc_commit(smem_u32(&bars->dp_full));
      tc_commit(smem_u32(&bars->drain));
      mbar_wait_drain(smem_u32(&bars->drain), 0, budget);
    }
  } else if (warp == 2) {
    // ================= dX reduction issuer: each staged chunk goes to L2 as a TMA
    // reduce-add; up to NB - 1 stay in flight, and a buffer is released once the
    // reduction that read it has finished reading
    if (lane == 0 && ta < tb) {
      tma_prefetch_desc(&tmap_dx);
      TileIter it;
      it.init(tile_start, offsets, R, ta, tb);
      int n = 0;
      bool ok = true;
      for (; ok && it.valid(); it.next()) {
        const int y = (int)it.t0();
        for (int c = 0; c < D / 16; ++c, ++n) {
          const int b = n % NB;
          if (!mbar_wait(smem_u32(&bars->stg_full[b]), (uint32_t)((n / NB) & 1), status, budget)) {
            ok = false;
            break;
          }
          tma_reduce_add_2d(&tmap_dx, c * 16, y, sbase + L::oStg + b * kStg);
          bulk_commit();
          bulk_wait_read<NB - 1>();
          if (n >= NB - 1) mbar_arrive(smem_u32(&bars->stg_free[(n - (NB - 1)) % NB]));
        }
      }
      bulk_wait_all();
    }
  } else if (warp >= 4 && warp < 12) {
    // ================= elementwise warpgroups: thread = token row = TMEM lane; warpgroup
    // hh takes prototypes [64 hh, 64 hh + 64) of the slice
    const int hh = (warp >> 2) - 1;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const bool leader = threadIdx.x == 128;
    const int c0 = hh * 64;
    const int ncols = min(64, max(0, k_valid - pbase - c0));  // valid prototypes of this half
    uint8_t* arow = smem + L::oA + hh * kBoxB + r * 128;
    uint8_t* drow = smem + L::oDS + hh * kBoxB + r * 128;
    float* dloc = reinterpret_cast<float*>(smem + L::oDh);
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
      if (!mbar_wait_warp(smem_u32(&bars->sS_full), (uint32_t)(i & 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 1a: A = 2^(S log2 e - lse2), 16 prototypes at a time, back into TMEM as bf16
      // pairs (8 columns per chunk) over S columns this thread has already read; runs while
      // the tensor pipe computes dA'
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = c0 + c * 16;
        uint32_t s16[16], ap[8];
        tmem_ld16(tmem + lane_off + kColS + col, s16);
        tmem_wait16(s16);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int x = 2 * q;
          const float a0 = (valid && c * 16 + x < ncols)
                               ? ex2_approx(fmaf(__uint_as_float(s16[x]), 1.4426950408889634f, -l2))
                               : 0.f;
          const float a1 = (valid && c * 16 + x + 1 < ncols)
                               ? ex2_approx(fmaf(__uint_as_float(s16[x + 1]), 1.4426950408889634f, -l2))
                               : 0.f;
          ap[q] = cvt_bf16x2(a0, a1);
        }
        tmem_st8(tmem + lane_off + kColS + c0 + c * 8, ap);
      }
      tmem_wait_st();
      if (!mbar_wait_warp(smem_u32(&bars->sG_full), (uint32_t)(i & 1), status, budget) ||
          (first && !mbar_wait_warp(smem_u32(&bars->g_full), (uint32_t)(seg & 1), status, budget))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 1b: this half's part of D = sum_j A (dA' - c), with A as the bf16 the MMAs use
      float dsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = c0 + c * 16;
        uint32_t g16[16], ap[8];
        tmem_ld16(tmem + lane_off + kColG + col, g16);
        tmem_ld8(tmem + lane_off + kColS + c0 + c * 8, ap);
        tmem_wait16(g16);
        tmem_wait8(ap);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 cv = *reinterpret_cast<const float4*>(csm + col + 4 * q);
          const uint32_t p0 = ap[2 * q], p1 = ap[2 * q + 1];
          dsum = fmaf(__uint_as_float(p0 << 16), __uint_as_float(g16[4 * q]) - cv.x, dsum);
          dsum = fmaf(__uint_as_float(p0 & 0xFFFF0000u), __uint_as_float(g16[4 * q + 1]) - cv.y, dsum);
          dsum = fmaf(__uint_as_float(p1 << 16), __uint_as_float(g16[4 * q + 2]) - cv.z, dsum);
          dsum = fmaf(__uint_as_float(p1 & 0xFFFF0000u), __uint_as_float(g16[4 * q + 3]) - cv.w, dsum);
        }
      }
      // the two halves meet in warpgroup 0, which sends D's partial to every CTA of the
      // cluster (4 tokens per st.async)
      const int qs = i % NX;
      const uint32_t xbar = smem_u32(&bars->xch[qs]);
      if (hh == 1) {
        dloc[r] = dsum;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->dhalf));
      } else {
        if (!mbar_wait_warp(smem_u32(&bars->dhalf), (uint32_t)(i & 1), status, budget)) {
          ok = false;
          break;
        }
        dsum += dloc[r];
        const int g0 = lane & ~3;
        const float v0 = __shfl_sync(0xffffffffu, dsum, g0 + 0);
        const float v1 = __shfl_sync(0xffffffffu, dsum, g0 + 1);
        const float v2 = __shfl_sync(0xffffffffu, dsum, g0 + 2);
        const float v3 = __shfl_sync(0xffffffffu, dsum, g0 + 3);
        const uint32_t laddr = smem_u32(xch + ((qs * C + (int)rank) * 128 + q4 * 32 + g0));
        for (int p = lane & 3; p < C; p += 4)
          st_async_v4(mapa(laddr, (uint32_t)p), v0, v1, v2, v3, mapa(xbar, (uint32_t)p));
        if (leader) mbar_arrive_expect_tx(xbar, (uint32_t)C * 512u);
      }
      if (!mbar_wait_warp<true>(xbar, (uint32_t)((i / NX) & 1), status, budget)) {
        ok = false;
        break;
      }
      float Dt = 0.f;
      for (int p = 0; p < C; ++p) Dt += xch[(qs * C + p) * 128 + r];  // fixed order
      // dX_part(i - 1) and dPn's MMA of tile i - 1 have read the A and dS tiles
      if (i > 0 && !mbar_wait_warp(smem_u32(&bars->tiles_free), (uint32_t)((i - 1) & 1), status, budget)) {
        ok = false;
        break;
      }
      // pass 2: dS = A (dA' - c - D) from pass 1's A (TMEM, bf16 pairs) and a second read of
      // dA'; A and dS as bf16 into their tiles, 16 prototypes (two 16-byte chunks of a row)
      // at a time. The next chunk's TMEM loads are in flight while this one is computed.
      {
        uint32_t gA[16], aA[8], gB[16], aB[8];
        auto load = [&](int c, uint32_t (&g)[16], uint32_t (&a)[8]) {
          tmem_ld16(tmem + lane_off + kColG + c0 + c * 16, g);
          tmem_ld8(tmem + lane_off + kColS + c0 + c * 8, a);
        };
        auto body = [&](int c, uint32_t (&g)[16], uint32_t (&ap)[8]) {
          const int col = c0 + c * 16;
          uint32_t pd[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 cv = *reinterpret_cast<const float4*>(csm + col + 4 * q);
            const uint32_t p0 = ap[2 * q], p1 = ap[2 * q + 1];
            const float d0 = __uint_as_float(p0 << 16) * (__uint_as_float(g[4 * q]) - (cv.x + Dt));
            const float d1 = __uint_as_float(p0 & 0xFFFF0000u) * (__uint_as_float(g[4 * q + 1]) - (cv.y + Dt));
            const float d2 = __uint_as_float(p1 << 16) * (__uint_as_float(g[4 * q + 2]) - (cv.z + Dt));
            const float d3 = __uint_as_float(p1 & 0xFFFF0000u) * (__uint_as_float(g[4 * q + 3]) - (cv.w + Dt));
            pd[2 * q] = cvt_bf16x2(d0, d1);
            pd[2 * q + 1] = cvt_bf16x2(d2, d3);
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int ch = c * 2 + h2;  // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4*>(arow + ((ch ^ (r & 7)) << 4)) =
                make_uint4(ap[4 * h2], ap[4 * h2 + 1], ap[4 * h2 + 2], ap[4 * h2 + 3]);
            *reinterpret_cast<uint4*>(drow + ((ch ^ (r & 7)) << 4)) =
                make_uint4(pd[4 * h2], pd[4 * h2 + 1], pd[4 * h2 + 2], pd[4 * h2 + 3]);
          }
        };
        load(0, gA, aA);
        tmem_wait16(gA);
        tmem_wait8(aA);
        load(1, gB, aB);
        body(0, gA, aA);
        tmem_wait16(gB);
        tmem_wait8(aB);
        load(2, gA, aA);
        body(1, gB, aB);
        tmem_wait16(gA);
        tmem_wait8(aA);
        load(3, gB, aB);
        body(2, gA, aA);
        tmem_wait16(gB);
        tmem_wait8(aB);
        body(3, gB, aB);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full));
    }
  } else if (warp >= 12) {
    // ================= dX epilogue: TMEM -> shared staging (16-column chunks, NB buffers);
    // warp 2 issues the TMA reduce-adds into dX
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    TileIter it;
    it.init(tile_start, offsets, R, ta, tb);
    int i = 0, n = 0;  // n: staging chunks filled so far (buffer n % NB, phase n / NB)
    bool ok = true;
    for (; ok && it.valid(); it.next(), ++i) {
      if (!mbar_wait_warp(smem_u32(&bars->dx_full), (uint32_t)(i & 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int h = 0; ok && h < D / 32; ++h) {
        uint32_t v[32];
        tmem_ld32_raw(tmem + lane_off + kColX + h * 32, v);
        tmem_wait_tie(v);
        if (h == D / 32 - 1) {  // dX_part fully read: TMEM is free for the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->dx_empty));
        }
#pragma unroll
        for (int half = 0; half < 2; ++half, ++n) {
          const int b = n % NB;
          // the reduction that last used this buffer has finished reading it
          if (n >= NB && !mbar_wait_warp(smem_u32(&bars->stg_free[b]), (uint32_t)((n / NB - 1) & 1),
                                         status, budget)) {
            ok = false;
            break;
          }
          // 64-byte rows with the 64B swizzle: 16-byte chunk x of row r sits at
          // x ^ ((r >> 1) & 3), so a quarter warp's 8 rows hit 8 different bank groups
          uint8_t* rowp = smem + L::oStg + b * kStg + r * 64;
#pragma unroll
          for (int x = 0; x < 4; ++x)
            *reinterpret_cast<float4*>(rowp + ((x ^ ((r >> 1) & 3)) << 4)) =
                make_float4(__uint_as_float(v[half * 16 + 4 * x]), __uint_as_float(v[half * 16 + 4 * x + 1]),
                            __uint_as_float(v[half * 16 + 4 * x + 2]),
                            __uint_as_float(v[half * 16 + 4 * x + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->stg_full[b]));
        }
      }
    }
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

template <int D, int NX, int NB>
cudaError_t configure_t(int C, size_t* smem) {
  auto kern = sa_bwd_fused_kernel<D, NX, NB>;
  *smem = smem_bytes_t<D, NX, NB>(C);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)*smem);
  if (e != cudaSuccess) return e;
  if (C > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int D, int NX, int NB>
cudaError_t max_clusters_t(int C, int* n) {
  size_t smem = 0;
  cudaError_t e = configure_t<D, NX, NB>(C, &smem);
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
  return cudaOccupancyMaxActiveClusters(n, sa_bwd_fused_kernel<D, NX, NB>, &cfg);
}

// Row-major [rows, cols] tensor maps: bf16 operands in 64-column boxes of 128 rows with
// the 128-byte swizzle; the fp32 dX in 16-column boxes of 128 rows with the 64-byte one.
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
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NX, int NB>
cudaError_t launch_t(const BwdFusedArgs& a, cudaStream_t s) {
  CUtensorMap tx, tpn, tgh, tdx;
  if (!map_bf16(&tx, a.X, (uint64_t)a.n_total, a.d) || !map_bf16(&tpn, a.pn, (uint64_t)a.k_pad, a.d) ||
      !map_bf16(&tgh, a.gh, (uint64_t)a.R * a.k_pad, a.d) ||
      !map_f32_rows(&tdx, a.dX, (uint64_t)a.n_total, a.d))
    return cudaErrorInvalidValue;
  size_t smem = 0;
  cudaError_t e = configure_t<D, NX, NB>(a.C, &smem);
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
  return cudaLaunchKernelEx(&cfg, sa_bwd_fused_kernel<D, NX, NB>, tx, tpn, tgh, tdx, a.offsets, a.R,
                            a.k_valid, a.C, a.k_pad, a.hdr, a.tile_start, a.lse, a.lse_scale, a.cj,
                            a.dpp_part, a.budget);
}

}  // namespace

// Exchange slots: 2 (tiles are handled in order, so a slot is read by both elementwise
// warpgroups before any CTA can send the tile two ahead into it). Staging buffers: 3
// while shared memory has room (clusters of up to 8), else 2.
cudaError_t bwd_fused_max_clusters(int d, int C, int* n) {
  if (d == 64) return C <= 8 ? max_clusters_t<64, 2, 3>(C, n) : max_clusters_t<64, 2, 2>(C, n);
  return C <= 8 ? max_clusters_t<128, 2, 3>(C, n) : max_clusters_t<128, 2, 2>(C, n);
}

cudaError_t launch_bwd_fused(const BwdFusedArgs& a, cudaStream_t s) {
  if (a.d == 64) return a.C <= 8 ? launch_t<64, 2, 3>(a, s) : launch_t<64, 2, 2>(a, s);
  return a.C <= 8 ? launch_t<128, 2, 3>(a, s) : launch_t<128, 2, 2>(a, s);
}

}  // namespace sa
