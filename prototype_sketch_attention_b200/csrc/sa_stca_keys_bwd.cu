// Backward of the ragged-key cross attention (the recent branch of STCA, "100,000 videos
// in your pocket" blog, section "2. STCA reasons at two time scales") on tcgen05, sm_100a.
//
// With the forward's Q' = Q W_q W_K^T log2(e) / sqrt(d) (bf16 hi + lo), lse2 and O'
// (recomputed before this kernel), dO' = dL/dO' = G W_V^T (bf16) and D_c = dO'_c . O'_c,
// every (candidate c, key row j) pair of a user contributes
//   a_cj  = 2^(Q'_c . Kx_j - lse2_c)               the attention weight
//   dz_cj = a_cj (dO'_c . Kx_j - D_c)              dL/d(score), natural units
//   G1_c  += dz_cj Kx_j                            (dQ = G1 M^T / sqrt(d) afterwards)
//   dKx_j += dz_cj Qn_c + a_cj dO'_c,  Qn = Q' ln 2.
//
// One CTA per (user, 128-candidate tile), walking the user's key tiles like the forward.
// Per key tile j:
//   S = (Q'_hi + Q'_lo) Kx_j^T and dP = dO' Kx_j^T on the tensor cores (TMEM, candidate =
//   lane); two elementwise warpgroups (64 key columns each, thread = candidate) form
//   a and dz, park them as bf16 pairs in TMEM over the dP columns they read (so the next
//   tile's score MMAs can start), and once the previous tile's MMAs have read the shared
//   dz / a tiles, store dz and a log2(e) there as bf16 [candidate][key] tiles;
//   then G1 += dz Kx_j (dz K-major, Kx_j MN-major) accumulates in TMEM over the whole walk,
//   and dKx_part = dz^T Q'_hi + (a log2 e)^T dO' (both A operands MN-major, K = the
//   candidates) goes to TMEM, from where an epilogue warpgroup adds ln(2) dKx_part into
//   dKx in global memory with vector reductions at L2, regrouped by warp shuffles so that
//   each reduction instruction covers whole 128-byte row segments (the user's candidate
//   tiles, and users whose ranges overlap, meet there). G1 is written once at the end (each candidate tile
//   has one owner).
// Roles: warp 0 TMA (the candidate tile's Q'_hi, Q'_lo and dO' once, the key tiles in a
// ring), warp 1 TMEM allocation and every MMA, warps 2-9 the elementwise step, warps
// 10-13 the dKx epilogue (a warp reads the TMEM lanes of quadrant warp mod 4). Every
// mbarrier wait is bounded.
#include <cuda.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kBox = 16384;  // 128 rows x 128 bytes (64 bf16), 128B swizzle
constexpr int kThreads = 448;  // 14 warps; at most 128 registers each, since a sub-partition
                               // (16,384 registers) hosts four of them
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 128, kColG = 256, kColK = 384;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory (every MMA operand block 1024-byte aligned):
//   Q'_hi, Q'_lo, dO'  (d/64) boxes each: the candidate tile, loaded once
//   key ring           NK x (d/64) boxes
//   dz, a log2(e)      two 16 KB boxes each ([candidate][64 keys]): K-major A of G1 += dz Kx,
//                      MN-major A of dKx_part (M = the key rows)
template <int D>
struct BSmem {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTile = kBoxes * kBox;
  static constexpr int kNK = D == 128 ? 2 : 3;  // 7 x 32 KB at d = 128
  static constexpr int oQh = 0;
  static constexpr int oQl = kTile;
  static constexpr int oDO = 2 * kTile;
  static constexpr int oK = 3 * kTile;
  static constexpr int oDZ = oK + kNK * kTile;
  static constexpr int oA = oDZ + 2 * kBox;
  static constexpr int oBars = oA + 2 * kBox;
};

struct BBars {
  uint64_t q_full, k_full[3], k_empty[3];
  uint64_t sd_full, s_empty, p_empty, ew_full, ew_empty, dk_full, dk_empty;
  uint64_t drain;
  uint32_t tmem_base;
};

// One stage of a butterfly that regroups a warp's 32 x 32 block (lane = row, register =
// column): lanes l and l ^ 2^LB swap the 4-register groups whose index bit GB differs from
// lane bit LB. After the stages (LB, GB) = (4, 2), (3, 1), (2, 0), register group s of
// lane l holds row 4 s + (l mod 4), columns 4 (l / 4) .. 4 (l / 4) + 3, so one vector
// reduction over the warp covers 4 rows x 128 contiguous bytes.
template <int LB, int GB>
__device__ __forceinline__ void regroup_stage(float (&v)[32], int lane) {
  const bool hi = (lane >> LB) & 1;
#pragma unroll
  for (int gi = 0; gi < 8; ++gi) {
    if ((gi >> GB) & 1) continue;
    const int gj = gi | (1 << GB);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float send = hi ? v[4 * gi + c] : v[4 * gj + c];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1 << LB);
      if (hi) v[4 * gi + c] = recv; else v[4 * gj + c] = recv;
    }
  }
}

// dst[0..3] += v (fp32, one vector reduction performed at L2)
__device__ __forceinline__ void red_add_v4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
               ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
stca_keys_bwd_kernel(const __grid_constant__ CUtensorMap tmap_qh,
                     const __grid_constant__ CUtensorMap tmap_ql,
                     const __grid_constant__ CUtensorMap tmap_do,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const int64_t* __restrict__ coff, const int64_t* __restrict__ kb,
                     const int64_t* __restrict__ ke, int R, const WsHeader* hdr_c,
                     const long long* __restrict__ tile_start, const float* __restrict__ lse2,
                     const float* __restrict__ Dd, float* __restrict__ G1,
                     float* __restrict__ dKx, long long budget) {
  using L = BSmem<D>;
  constexpr int KS_D = D / 16;
  constexpr int NK = L::kNK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  BBars* bars = reinterpret_cast<BBars*>(smem + L::oBars);
  WsHeader* hdr = const_cast<WsHeader*>(hdr_c);
  int* status = &hdr->status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const long long g = blockIdx.x;
  if (__syncthreads_or(read_status(status) != 0) || g >= hdr->total_tiles) return;
  const int u = user_of_tile(tile_start, R, g);
  const long long c0 = coff[u] + (g - tile_start[u]) * 128;
  const int nv = (int)min(128LL, coff[u + 1] - c0);
  const long long k0 = kb[u], k1 = ke[u];
  const int nkt = (int)((k1 - k0 + 127) / 128);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->sd_full), 1);
    mbar_init(smem_u32(&bars->s_empty), 8);
    mbar_init(smem_u32(&bars->p_empty), 8);
    mbar_init(smem_u32(&bars->ew_full), 8);
    mbar_init(smem_u32(&bars->ew_empty), 1);
    mbar_init(smem_u32(&bars->dk_full), 1);
    mbar_init(smem_u32(&bars->dk_empty), 4);
    mbar_init(smem_u32(&bars->drain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ================= TMA
    if (lane == 0 && nkt > 0) {
      tma_prefetch_desc(&tmap_qh);
      tma_prefetch_desc(&tmap_ql);
      tma_prefetch_desc(&tmap_do);
      tma_prefetch_desc(&tmap_k);
      const uint32_t qf = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qf, 3 * L::kTile);
      for (int b = 0; b < L::kBoxes; ++b) {
        tma_load_2d(sbase + L::oQh + b * kBox, &tmap_qh, b * 64, (int)c0, qf);
        tma_load_2d(sbase + L::oQl + b * kBox, &tmap_ql, b * 64, (int)c0, qf);
        tma_load_2d(sbase + L::oDO + b * kBox, &tmap_do, b * 64, (int)c0, qf);
      }
      int j = 0;
      for (; j < nkt; ++j) {
        const int st = j % NK;
        if (!mbar_wait(smem_u32(&bars->k_empty[st]), (uint32_t)(((j / NK) & 1) ^ 1), status, budget)) break;
        const uint32_t fb = smem_u32(&bars->k_full[st]);
        mbar_arrive_expect_tx(fb, L::kTile);
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_2d(sbase + L::oK + st * L::kTile + b * kBox, &tmap_k, b * 64, (int)(k0 + 128LL * j), fb);
      }
      for (int i = (j > NK ? j - NK : 0); i < j; ++i)
        mbar_wait_drain(smem_u32(&bars->k_full[i % NK]), (uint32_t)((i / NK) & 1), budget);
      mbar_wait_drain(qf, 0, budget);
    }
  } else if (warp == 1) {
    // ================= MMAs, in order: S(j), dP(j), then G1 and dKx_part of tile j - 1
    if (lane == 0 && nkt > 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);  // [cand x d] (K) x Kx (K)
      const uint32_t id_g = idesc_bf16_f32(128, D, 0, 1);    // dz (K) x Kx (MN)
      const uint32_t id_k = idesc_bf16_f32(128, D, 1, 1);    // dz^T (MN) x Q'_hi / dO' (MN)
      const uint64_t dqh = smem_desc(sbase + L::oQh, 16, 1024, kSwizzle128B);
      const uint64_t dql = smem_desc(sbase + L::oQl, 16, 1024, kSwizzle128B);
      const uint64_t ddo = smem_desc(sbase + L::oDO, 16, 1024, kSwizzle128B);
      const uint64_t dqh_mn = smem_desc(sbase + L::oQh, kBox, 1024, kSwizzle128B);
      const uint64_t ddo_mn = smem_desc(sbase + L::oDO, kBox, 1024, kSwizzle128B);
      const uint64_t ddz_k = smem_desc(sbase + L::oDZ, 16, 1024, kSwizzle128B);
      const uint64_t ddz_mn = smem_desc(sbase + L::oDZ, kBox, 1024, kSwizzle128B);
      const uint64_t da_mn = smem_desc(sbase + L::oA, kBox, 1024, kSwizzle128B);
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0, status, budget);
      auto back = [&](int i) {  // G1 += dz(i) Kx_i; dKx_part = dz(i)^T Q'_hi + a'(i)^T dO'
        const int st = i % NK;
        ok = ok && mbar_wait(smem_u32(&bars->ew_full), (uint32_t)(i & 1), status, budget);
        if (!ok) return;
        tc_fence_after();
        const uint64_t dk_mn = smem_desc(sbase + L::oK + st * L::kTile, kBox, 1024, kSwizzle128B);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc_mma_f16(tmem + kColG, ddz_k + (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4),
                     dk_mn + (uint64_t)((ks * 2048) >> 4), id_g, (i > 0 || ks > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bars->k_empty[st]));
        ok = mbar_wait(smem_u32(&bars->dk_empty), (uint32_t)((i & 1) ^ 1), status, budget);
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc_mma_f16(tmem + kColK, ddz_mn + (uint64_t)((ks * 2048) >> 4),
                     dqh_mn + (uint64_t)((ks * 2048) >> 4), id_k, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc_mma_f16(tmem + kColK, da_mn + (uint64_t)((ks * 2048) >> 4),
                     ddo_mn + (uint64_t)((ks * 2048) >> 4), id_k, 1u);
        tc_commit(smem_u32(&bars->dk_full));
        tc_commit(smem_u32(&bars->ew_empty));
      };
      for (int j = 0; ok && j < nkt; ++j) {
        const int st = j % NK;
        ok = mbar_wait(smem_u32(&bars->k_full[st]), (uint32_t)((j / NK) & 1), status, budget) &&
             (j == 0 || mbar_wait(smem_u32(&bars->s_empty), (uint32_t)((j - 1) & 1), status, budget));
        if (!ok) break;
        tc_fence_after();
        const uint64_t dk = smem_desc(sbase + L::oK + st * L::kTile, 16, 1024, kSwizzle128B);
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
          const uint64_t koff = (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4);
          tc_mma_f16(tmem + kColS, dqh + koff, dk + koff, id_s, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
          const uint64_t koff = (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4);
          tc_mma_f16(tmem + kColS, dql + koff, dk + koff, id_s, 1u);
        }
        // dP(j) once the elementwise step has moved the previous tile's packed dz and a out
        // of the dP columns
        ok = j == 0 || mbar_wait(smem_u32(&bars->p_empty), (uint32_t)((j - 1) & 1), status, budget);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
          const uint64_t koff = (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4);
          tc_mma_f16(tmem + kColP, ddo + koff, dk + koff, id_s, ks > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&bars->sd_full));
        if (j > 0) back(j - 1);
      }
      if (ok) back(nkt - 1);
      tc_commit(smem_u32(&bars->drain));
      mbar_wait_drain(smem_u32(&bars->drain), 0, budget);
    }
  } else if (warp >= 2 && warp < 10) {
    // ================= elementwise: thread = candidate row, warpgroup w = key columns
    // [64w, 64w + 64); warps 2-5 and 6-9 each cover the four TMEM lane quadrants
    const int w = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const bool row_ok = r < nv;
    const float l2 = row_ok ? lse2[c0 + r] : 0.f;
    const float dc = row_ok ? Dd[c0 + r] : 0.f;
    uint8_t* dzrow = smem + L::oDZ + w * kBox + r * 128;
    uint8_t* arow = smem + L::oA + w * kBox + r * 128;
    bool ok = true;
    for (int j = 0; ok && j < nkt; ++j) {
      const int nk = (int)min(128LL, k1 - k0 - 128LL * j);
      if (!mbar_wait_warp(smem_u32(&bars->sd_full), (uint32_t)(j & 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // dz and a log2(e) of this thread's 64 key columns as bf16 pairs, 16 columns at a
      // time, written back into TMEM over the dP columns just read (8 + 8 per 16 columns)
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        const int col = 64 * w + 16 * q;
        uint32_t sv[16], pv[16], pk[16];
        tmem_ld16(tmem + lane_off + kColS + col, sv);
        tmem_ld16(tmem + lane_off + kColP + col, pv);
        tmem_wait16(sv);
        tmem_wait16(pv);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const bool v0 = row_ok && col + 2 * x < nk, v1 = row_ok && col + 2 * x + 1 < nk;
          const float a0 = v0 ? ex2_approx(__uint_as_float(sv[2 * x]) - l2) : 0.f;
          const float a1 = v1 ? ex2_approx(__uint_as_float(sv[2 * x + 1]) - l2) : 0.f;
          pk[x] = cvt_bf16x2(a0 * (__uint_as_float(pv[2 * x]) - dc),
                             a1 * (__uint_as_float(pv[2 * x + 1]) - dc));
          pk[8 + x] = cvt_bf16x2(a0 * kLog2e, a1 * kLog2e);
        }
        tmem_st16(tmem + lane_off + kColP + col, pk);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      // S is read: the next tile's score MMAs may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty));
      // the previous tile's G1 and dKx MMAs have read dz and a: store this tile's
      if (!mbar_wait_warp(smem_u32(&bars->ew_empty), (uint32_t)((j & 1) ^ 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[16];
        tmem_ld16(tmem + lane_off + kColP + 64 * w + 16 * q, pk);
        tmem_wait16(pk);
        const int o0 = ((2 * q) ^ (r & 7)) << 4, o1 = ((2 * q + 1) ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(dzrow + o0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dzrow + o1) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        *reinterpret_cast<uint4*>(arow + o0) = make_uint4(pk[8], pk[9], pk[10], pk[11]);
        *reinterpret_cast<uint4*>(arow + o1) = make_uint4(pk[12], pk[13], pk[14], pk[15]);
      }
      // the dP columns are free for the next tile's dP MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_empty));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->ew_full));
    }
    // ---- G1 of this candidate tile: complete once the last tile's MMAs are
    const bool have = ok && nkt > 0 &&
                      mbar_wait_warp(smem_u32(&bars->ew_empty), (uint32_t)((nkt - 1) & 1), status, budget);
    if (have) tc_fence_after();
    float* grow = G1 + (c0 + r) * D;
#pragma unroll 1
    for (int c = w * (D / 64); c < (w + 1) * (D / 64); ++c) {  // this warpgroup's half of d
      uint32_t v[32];
      if (have) {
        tmem_ld32_raw(tmem + lane_off + kColG + 32 * c, v);
        tmem_wait_tie(v);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int x = 0; x < 32; x += 4)
          *reinterpret_cast<float4*>(grow + 32 * c + x) =
              make_float4(__uint_as_float(v[x]), __uint_as_float(v[x + 1]),
                          __uint_as_float(v[x + 2]), __uint_as_float(v[x + 3]));
      }
    }
  } else {
    // ================= dKx epilogue: dKx += ln(2) dKx_part, warp = 32 key rows of the tile
    // (TMEM lane quadrant warp mod 4), regrouped so that each reduction is coalesced
    const int q4 = warp & 3;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bool ok = true;
    for (int j = 0; ok && j < nkt; ++j) {
      const int nk = (int)min(128LL, k1 - k0 - 128LL * j);
      ok = mbar_wait_warp(smem_u32(&bars->dk_full), (uint32_t)(j & 1), status, budget);
      if (!ok) break;
      tc_fence_after();
      float* dtile = dKx + (k0 + 128LL * j + q4 * 32) * D;  // this warp's 32 rows
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32_raw(tmem + lane_off + kColK + 32 * c, u);
        tmem_wait_tie(u);
        if (c == D / 32 - 1) {  // dKx_part of this tile has been read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->dk_empty));
        }
        float v[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = __uint_as_float(u[x]) * kLn2;
        regroup_stage<4, 2>(v, lane);
        regroup_stage<3, 1>(v, lane);
        regroup_stage<2, 0>(v, lane);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int row = 4 * g + (lane & 3);  // within the warp's 32 rows
          if (q4 * 32 + row < nk)
            red_add_v4(dtile + row * D + 32 * c + 4 * (lane >> 2), v[4 * g], v[4 * g + 1],
                       v[4 * g + 2], v[4 * g + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_t(const StcaKeysBwdArgs& a, cudaStream_t s) {
  CUtensorMap tqh, tql, tdo, tk;
  if (!tmap_rows_bf16(&tqh, a.Qh, (uint64_t)a.n_cand, D) ||
      !tmap_rows_bf16(&tql, a.Ql, (uint64_t)a.n_cand, D) ||
      !tmap_rows_bf16(&tdo, a.dOb, (uint64_t)a.n_cand, D) ||
      !tmap_rows_bf16(&tk, a.Kx, (uint64_t)a.n_keys, D))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + BSmem<D>::oBars + sizeof(BBars);
  cudaError_t e = cudaFuncSetAttribute(stca_keys_bwd_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = a.n_cand / 128 + a.R + 1;  // bounds the candidate tiles; the rest exit
  stca_keys_bwd_kernel<D><<<(unsigned)grid, kThreads, smem, s>>>(
      tqh, tql, tdo, tk, a.coff, a.kb, a.ke, a.R, a.hdr, a.tile_start, a.lse2, a.Dd, a.G1, a.dKx,
      kDefaultWaitBudget);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stca_keys_bwd_kernel(const StcaKeysBwdArgs& a, cudaStream_t s) {
  if (a.n_cand == 0 || a.n_keys == 0) return cudaSuccess;
  return a.d == 64 ? launch_t<64>(a, s) : launch_t<128>(a, s);
}

}  // namespace sa
