// Cross attention from each user's candidates to a ragged set of that user's key rows, on
// tcgen05 (sm_100a): the recent branch of STCA, whose keys are the user's most recent
// raw history tokens ("100,000 videos in your pocket" blog, section "2. STCA reasons at
// two time scales", recent branch: the candidate attends over the last 10K tokens).
//
// User u's candidates c in [coff[u], coff[u+1]) attend over the key rows
// Kx[kb[u] : ke[u]] (for the recent branch, Kx is the history X itself and the range is
// the last min(n_u, L) tokens, so nothing is copied). With the same refold as the sketch
// branch, Q' = Q W_q W_K^T log2(e) / sqrt(d) (computed before this kernel):
//   z_cj = Q'_c . Kx_j (log2 units),  a_cj = 2^(z_cj - lse2_c),  O'_c = sum_j a_cj Kx_j,
// and out = O' W_V afterwards. Keys and values are the same rows, so one TMA tile of 128
// key rows is the B operand of both MMAs: K-major for Z = Q' Kx^T, MN-major for
// O' += P Kx. Q' is formed in fp32 and enters the score MMA as a bf16 pair hi + lo (two
// accumulated MMAs, about 16 significant bits): with scores of tens of units a single bf16
// rounding of Q' would move the weights by several percent.
//
// One CTA per (user, 128-candidate tile). Two softmax warpgroups take alternate key tiles
// (warpgroup w the tiles j with j mod 2 = w), each with its own score buffer Z_w, P
// buffer and accumulator O'_w in TMEM, and its own running maximum m_w and sum l_w along
// each candidate's row (one thread per candidate = TMEM lane). The running maximum is
// raised only when a tile's maximum exceeds it by more than 8 (in log2 units): then O'_w
// and l_w are rescaled once; otherwise the exponentials stay below 2^8. P = 2^(z - m_w)
// goes to shared memory as bf16 (the K-major A operand of O'_w += P Kx). At the end the
// two halves merge: m = max(m_0, m_1), O' = (O'_0 2^(m_0 - m) + O'_1 2^(m_1 - m)) / l and
// lse2 = m + log2 l with l = l_0 2^(m_0 - m) + l_1 2^(m_1 - m).
// Roles: warp 0 TMA, warp 1 TMEM allocation and the MMAs, warps 4-7 and 8-11 the softmax
// warpgroups (warpgroup 0 also merges and writes the output). Every mbarrier wait is
// bounded.
//
// The backward (launch_stca_keys_backward) recomputes this forward, forms dO' = G W_V^T and
// dW_V = O'^T G on the tcgen05 GEMM, then runs its own tcgen05 kernel (sa_stca_keys_bwd.cu)
// for G1 = dL/dQn and dKx, and finishes dQ, dW_q and dW_K with GEMMs.
#include <cuda.h>

#include <algorithm>
#include <cmath>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kBox = 16384;   // 128 rows x 128 bytes, 128B swizzle
constexpr int kNKMax = 3;     // key stages
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: score buffers Z_0 at 0 and Z_1 at 128, accumulators O'_0 at 256 and O'_1
// at 384 (d <= 128 columns each)
__host__ __device__ constexpr uint32_t col_z(int w) { return w ? 128u : 0u; }
__host__ __device__ constexpr uint32_t col_o(int w) { return w ? 384u : 256u; }
constexpr float kRescale = 8.f;  // raise the running max only when a tile exceeds it by this
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct KSmem {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTile = kBoxes * kBox;
  static constexpr int kNK = 3;  // at d = 128: 7 x 32 KB + 1 KB + barriers, within 227 KB
  static constexpr int oQ = 0;                 // Q' as bf16 hi, then lo
  static constexpr int oK = oQ + 2 * kTile;
  static constexpr int oP = oK + kNK * kTile;  // 2 buffers x two 64-key blocks
  static constexpr int oML = oP + 4 * kBox;    // warpgroup 1's m and l per row (merge)
  static constexpr int oBars = oML + 2 * 128 * 4;
};

struct KBars {
  uint64_t q_full, k_full[kNKMax], k_empty[kNKMax];
  uint64_t z_full[2], z_empty[2], p_full[2], p_empty[2];
  uint64_t merge, drain;
  uint32_t tmem_base;
};

// 64 consecutive TMEM columns of this warp's 32 lanes: two loads, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&a)[32], uint32_t (&b)[32]) {
  tmem_ld32_raw(taddr, a);
  tmem_ld32_raw(taddr + 32, b);
  tmem_wait_tie(a);
  tie32(b);
}

__device__ __forceinline__ void tmem_st32k(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
      " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
        "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
        "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 2^(z - m) of 16 scores as 8 bf16 pairs (0 for columns at or past nk), and their sum.
__device__ __forceinline__ float exp_pack16(const uint32_t* z, int col0, int nk, float m,
                                            uint32_t (&pk)[8]) {
  float s = 0.f;
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const float e0 = col0 + 2 * x < nk ? ex2_approx(__uint_as_float(z[2 * x]) - m) : 0.f;
    const float e1 = col0 + 2 * x + 1 < nk ? ex2_approx(__uint_as_float(z[2 * x + 1]) - m) : 0.f;
    s += e0 + e1;
    pk[x] = cvt_bf16x2(e0, e1);
  }
  return s;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
stca_keys_fwd_kernel(const __grid_constant__ CUtensorMap tmap_qh,
                     const __grid_constant__ CUtensorMap tmap_ql,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const int64_t* __restrict__ coff, const int64_t* __restrict__ kb,
                     const int64_t* __restrict__ ke, int R, const WsHeader* hdr_c,
                     const long long* __restrict__ tile_start, float* __restrict__ O,
                     float* __restrict__ lse2_out, float* __restrict__ lse_out, long long budget) {
  using L = KSmem<D>;
  constexpr int KS_D = D / 16;
  constexpr int kNK = L::kNK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  KBars* bars = reinterpret_cast<KBars*>(smem + L::oBars);
  WsHeader* hdr = const_cast<WsHeader*>(hdr_c);
  int* status = &hdr->status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's candidate tile: a user's tile of up to 128 candidates
  const long long g = blockIdx.x;
  if (__syncthreads_or(read_status(status) != 0) || g >= hdr->total_tiles) return;
  const int u = user_of_tile(tile_start, R, g);
  const long long c0 = coff[u] + (g - tile_start[u]) * 128;
  const int nv = (int)min(128LL, coff[u + 1] - c0);
  const long long k0 = kb[u], k1 = ke[u];
  const int nkt = (int)((k1 - k0 + 127) / 128);  // key tiles (0 for a user without keys)

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int s = 0; s < kNK; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->z_full[b]), 1);
      mbar_init(smem_u32(&bars->z_empty[b]), 4);
      mbar_init(smem_u32(&bars->p_full[b]), 4);
      mbar_init(smem_u32(&bars->p_empty[b]), 1);
    }
    mbar_init(smem_u32(&bars->merge), 4);
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
    // ================= TMA: the candidate tile of Q' (hi, lo) once, then the key tiles
    if (lane == 0 && nkt > 0) {
      tma_prefetch_desc(&tmap_qh);
      tma_prefetch_desc(&tmap_ql);
      tma_prefetch_desc(&tmap_k);
      const uint32_t qf = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qf, 2 * L::kTile);
      for (int b = 0; b < L::kBoxes; ++b) {
        tma_load_2d(sbase + L::oQ + b * kBox, &tmap_qh, b * 64, (int)c0, qf);
        tma_load_2d(sbase + L::oQ + L::kTile + b * kBox, &tmap_ql, b * 64, (int)c0, qf);
      }
      int j = 0;
      for (; j < nkt; ++j) {
        const int st = j % kNK;
        if (!mbar_wait(smem_u32(&bars->k_empty[st]), (uint32_t)(((j / kNK) & 1) ^ 1), status, budget)) break;
        const uint32_t fb = smem_u32(&bars->k_full[st]);
        mbar_arrive_expect_tx(fb, L::kTile);
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_2d(sbase + L::oK + st * L::kTile + b * kBox, &tmap_k, b * 64, (int)(k0 + 128LL * j), fb);
      }
      for (int i = (j > kNK ? j - kNK : 0); i < j; ++i)
        mbar_wait_drain(smem_u32(&bars->k_full[i % kNK]), (uint32_t)((i / kNK) & 1), budget);
      mbar_wait_drain(qf, 0, budget);
    }
  } else if (warp == 1) {
    // ================= MMAs: Z(j) = Q' Kx_j^T into Z_(j mod 2), then O'_(j mod 2) += P(j) Kx_j
    // once P(j) is stored; Z(j + 1) is issued before O'(j) so that the other warpgroup's
    // softmax of tile j + 1 runs while this one's P(j) is produced
    if (lane == 0 && nkt > 0) {
      const uint32_t id_z = idesc_bf16_f32(128, 128, 0, 0);  // Q' (K) x Kx (K)
      const uint32_t id_o = idesc_bf16_f32(128, D, 0, 1);    // P (K) x Kx (MN)
      const uint64_t dqh = smem_desc(sbase + L::oQ, 16, 1024, kSwizzle128B);
      const uint64_t dql = smem_desc(sbase + L::oQ + L::kTile, 16, 1024, kSwizzle128B);
      bool ok = mbar_wait(smem_u32(&bars->q_full), 0, status, budget);
      auto issue_z = [&](int j) {
        const int st = j % kNK, zb = j & 1;
        ok = ok && mbar_wait(smem_u32(&bars->k_full[st]), (uint32_t)((j / kNK) & 1), status, budget) &&
             mbar_wait(smem_u32(&bars->z_empty[zb]), (uint32_t)(((j >> 1) & 1) ^ 1), status, budget);
        if (!ok) return;
        tc_fence_after();
        const uint64_t dk = smem_desc(sbase + L::oK + st * L::kTile, 16, 1024, kSwizzle128B);
        // Z = (Q'_hi + Q'_lo) Kx^T: Q' enters at about 16 significant bits
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
          const uint64_t koff = (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4);
          tc_mma_f16(tmem + col_z(zb), dqh + koff, dk + koff, id_z, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
          const uint64_t koff = (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4);
          tc_mma_f16(tmem + col_z(zb), dql + koff, dk + koff, id_z, 1u);
        }
        tc_commit(smem_u32(&bars->z_full[zb]));
      };
      issue_z(0);
      for (int j = 0; ok && j < nkt; ++j) {
        if (j + 1 < nkt) issue_z(j + 1);
        const int st = j % kNK, pb = j & 1;
        ok = ok && mbar_wait(smem_u32(&bars->p_full[pb]), (uint32_t)((j >> 1) & 1), status, budget);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dp = smem_desc(sbase + L::oP + pb * 2 * kBox, 16, 1024, kSwizzle128B);
        const uint64_t dk = smem_desc(sbase + L::oK + st * L::kTile, kBox, 1024, kSwizzle128B);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc_mma_f16(tmem + col_o(pb), dp + (uint64_t)((((ks >> 2) * kBox) + (ks & 3) * 32) >> 4),
                     dk + (uint64_t)((ks * 2048) >> 4), id_o, (j >= 2 || ks > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bars->k_empty[st]));
        tc_commit(smem_u32(&bars->p_empty[pb]));  // P(j) read, and O'_(j mod 2) holds tile j
      }
      tc_commit(smem_u32(&bars->drain));
      mbar_wait_drain(smem_u32(&bars->drain), 0, budget);
    }
  } else if (warp >= 4) {
    // ================= softmax warpgroup w: key tiles j = w, w + 2, ...; thread = candidate
    const int w = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t zt = tmem + lane_off + col_z(w);
    const uint32_t ot = tmem + lane_off + col_o(w);
    uint8_t* prow0 = smem + L::oP + w * 2 * kBox + r * 128;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int last = -1;
    for (int j = w; ok && j < nkt; j += 2) {
      const int nk = (int)min(128LL, k1 - k0 - 128LL * j);  // valid keys of this tile
      if (!mbar_wait_warp(smem_u32(&bars->z_full[w]), (uint32_t)((j >> 1) & 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float mt = -INFINITY;  // this tile's row maximum over the valid keys
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t za[32], zb[32];
        tmem_ld64(zt + h * 64, za, zb);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          if (h * 64 + x < nk) mt = fmaxf(mt, __uint_as_float(za[x]));
          if (h * 64 + 32 + x < nk) mt = fmaxf(mt, __uint_as_float(zb[x]));
        }
      }
      // P(j - 2) has been read, and O'_w holds every earlier tile of this warpgroup
      if (!mbar_wait_warp(smem_u32(&bars->p_empty[w]), (uint32_t)(((j >> 1) & 1) ^ 1), status, budget)) {
        ok = false;
        break;
      }
      // raise the running max only past the margin; O'_w and l shrink by 2^(m - mt)
      const bool raise = mt > m + kRescale;
      if (__any_sync(0xffffffffu, raise)) {
        if (j >= 2) {
          tc_fence_after();
          const float f = raise ? ex2_approx(m - mt) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 64; ++c) {
            uint32_t oa[32], ob[32];
            tmem_ld64(ot + c * 64, oa, ob);
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              oa[x] = __float_as_uint(__uint_as_float(oa[x]) * f);
              ob[x] = __float_as_uint(__uint_as_float(ob[x]) * f);
            }
            tmem_st32k(ot + c * 64, oa);
            tmem_st32k(ot + c * 64 + 32, ob);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          l *= f;
        }
        if (raise) m = mt;
      }
      // P = 2^(z - m) (0 for keys past the range) as bf16 into the K-major P tile
      float ls = 0.f;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t za[32], zb[32];
        tmem_ld64(zt + h * 64, za, zb);
        uint8_t* prow = prow0 + h * kBox;  // keys [64h, 64h + 64): one 128-byte row
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[8];
          ls += exp_pack16((q < 2 ? za : zb) + (q & 1) * 16, h * 64 + q * 16, nk, m, pk);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int ch = q * 2 + hh;
            *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * hh], pk[4 * hh + 1], pk[4 * hh + 2], pk[4 * hh + 3]);
          }
        }
      }
      l += ls;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->z_empty[w]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[w]));
      last = j;
    }
    // ---- this warpgroup's accumulator is complete once its last O' MMA is
    if (ok && last >= 0)
      ok = mbar_wait_warp(smem_u32(&bars->p_empty[w]), (uint32_t)((last >> 1) & 1), status, budget);
    float* ml = reinterpret_cast<float*>(smem + L::oML);
    if (w == 1) {  // hand m_1 and l_1 to warpgroup 0
      ml[r] = m;
      ml[128 + r] = ok ? l : 0.f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->merge));
    } else {
      const bool merged = mbar_wait_warp(smem_u32(&bars->merge), 0, status, budget);
      const float m1 = ml[r], l1 = merged ? ml[128 + r] : 0.f;
      const float l0 = ok ? l : 0.f;
      const float mm = fmaxf(m, m1);
      const float f0 = l0 > 0.f ? ex2_approx(m - mm) : 0.f;
      const float f1 = l1 > 0.f ? ex2_approx(m1 - mm) : 0.f;
      const float lt = l0 * f0 + l1 * f1;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float g0 = f0 * inv, g1 = f1 * inv;
      if (nkt > 0) tc_fence_after();
      float* orow = O + (c0 + r) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t oa[32], ob[32];
        if (nkt > 0) {  // O'_0 (every user with keys has tile 0)
          tmem_ld32_raw(tmem + lane_off + col_o(0) + c * 32, oa);
          tmem_wait_tie(oa);
        }
        if (nkt > 1) {  // O'_1 only if warpgroup 1 had a tile
          tmem_ld32_raw(tmem + lane_off + col_o(1) + c * 32, ob);
          tmem_wait_tie(ob);
        }
        if (r < nv) {
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            float v[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const float a0 = nkt > 0 ? __uint_as_float(oa[x + y]) * g0 : 0.f;
              v[y] = nkt > 1 ? fmaf(__uint_as_float(ob[x + y]), g1, a0) : a0;
            }
            *reinterpret_cast<float4*>(orow + c * 32 + x) = make_float4(v[0], v[1], v[2], v[3]);
          }
        }
      }
      if (r < nv) {
        const float l2 = lt > 0.f ? mm + lg2_approx(lt) : -INFINITY;
        lse2_out[c0 + r] = l2;
        if (lse_out) lse_out[c0 + r] = l2 * kLn2;
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

// Output of users whose candidates see no key rows, when there are no key rows at all:
// O' = 0 and lse = -inf.
__global__ void keys_empty_kernel(long long n, int d, float* __restrict__ O, float* __restrict__ lse2,
                                  float* __restrict__ lse) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n * d;
       i += (long long)gridDim.x * blockDim.x) {
    O[i] = 0.f;
    if (i % d == 0) {
      lse2[i / d] = -INFINITY;
      if (lse) lse[i / d] = -INFINITY;
    }
  }
}

// M[f][e] = sum_g W_q[f][g] W_K[e][g] in fp32. Block b owns the rows f in [8b, 8b + 8):
// W_K goes to shared memory transposed ([g][e], fp32, rows padded by one), the block's
// W_q rows beside it, and thread e forms column e of those rows (conflict-free rows of
// W_K^T, broadcast W_q).
template <int D>
__global__ void __launch_bounds__(D) keys_mfold_kernel(const __nv_bfloat16* __restrict__ Wq,
                                                       const __nv_bfloat16* __restrict__ WK,
                                                       float* __restrict__ M) {
  extern __shared__ float fsm[];
  float* wkt = fsm;                  // [D][D + 1]: wkt[g][e] = W_K[e][g] (padded rows)
  float* wq = fsm + D * (D + 1);     // [8][D]
  const int e = threadIdx.x, f0 = blockIdx.x * 8;
  for (int i = e; i < D * D; i += D) wkt[(i % D) * (D + 1) + i / D] = __bfloat162float(WK[i]);
  for (int i = e; i < 8 * D; i += D) wq[i] = __bfloat162float(Wq[f0 * D + i]);
  __syncthreads();
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int g = 0; g < D; ++g) {
    const float w = wkt[g * (D + 1) + e];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = fmaf(wq[r * D + g], w, acc[r]);
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) M[(f0 + r) * D + e] = acc[r];
}

// Q'_c = scale Q_c M in fp32, stored as hi = bf16(Q'_c) and lo = bf16(Q'_c - hi). Each
// block keeps M in shared memory and walks groups of 32 candidates: their Q rows are
// staged in shared memory (fp32, padded), and thread t forms column t mod D of 32 / (256 / D)
// of the group's rows (broadcast Q, conflict-free rows of M).
template <int D>
__global__ void __launch_bounds__(256) keys_qfold_kernel(const __nv_bfloat16* __restrict__ Q,
                                                         const float* __restrict__ M, long long n,
                                                         float scale,
                                                         __nv_bfloat16* __restrict__ hi,
                                                         __nv_bfloat16* __restrict__ lo) {
  constexpr int kRows = 32, kPer = kRows * D / 256;  // rows per thread: 16 at d = 128
  extern __shared__ float fsm[];
  float* ms = fsm;               // [D][D]
  float* qs = fsm + D * D;       // [kRows][D + 1]
  const int t = threadIdx.x, e = t % D, r0 = (t / D) * kPer;
  for (int i = t; i < D * D; i += 256) ms[i] = M[i];
  for (long long c0 = (long long)blockIdx.x * kRows; c0 < n; c0 += (long long)gridDim.x * kRows) {
    __syncthreads();
    for (int i = t; i < kRows * D; i += 256) {
      const int r = i / D, f = i % D;
      qs[r * (D + 1) + f] = c0 + r < n ? __bfloat162float(Q[(c0 + r) * D + f]) : 0.f;
    }
    __syncthreads();
    float acc[kPer];
#pragma unroll
    for (int r = 0; r < kPer; ++r) acc[r] = 0.f;
    for (int f = 0; f < D; ++f) {
      const float m = ms[f * D + e];
#pragma unroll
      for (int r = 0; r < kPer; ++r) acc[r] = fmaf(qs[(r0 + r) * (D + 1) + f], m, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const long long c = c0 + r0 + r;
      if (c < n) {
        const float v = acc[r] * scale;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        hi[c * D + e] = h;
        lo[c * D + e] = __float2bfloat16_rn(v - __bfloat162float(h));
      }
    }
  }
}

template <int D>
cudaError_t launch_folds(const void* Wq, const void* WK, const void* Q, long long n, float scale,
                         float* M, __nv_bfloat16* Qh, __nv_bfloat16* Ql, cudaStream_t s) {
  const size_t m_smem = (size_t)(D * (D + 1) + 8 * D) * sizeof(float);
  const size_t q_smem = (size_t)(D * D + 32 * (D + 1)) * sizeof(float);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(keys_mfold_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)m_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(keys_qfold_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)q_smem)) != cudaSuccess)
    return e;
  keys_mfold_kernel<D><<<D / 8, D, m_smem, s>>>(static_cast<const __nv_bfloat16*>(Wq),
                                                static_cast<const __nv_bfloat16*>(WK), M);
  const long long groups = (n + 31) / 32;
  keys_qfold_kernel<D><<<(unsigned)std::min<long long>(groups, 148LL * 2), 256, q_smem, s>>>(
      static_cast<const __nv_bfloat16*>(Q), M, n, scale, Qh, Ql);
  return cudaGetLastError();
}

// D_c = sum_e bf16(dO'_ce) O'_ce, one warp per candidate.
__global__ void keys_rowdot_kernel(const __nv_bfloat16* __restrict__ dOb, const float* __restrict__ O,
                                   long long n, int d, float* __restrict__ D) {
  const int lane = threadIdx.x & 31;
  const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long c = w0; c < n; c += nw) {
    float acc = 0.f;
    for (int e = lane; e < d; e += 32) acc = fmaf(__bfloat162float(dOb[c * d + e]), O[c * d + e], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) D[c] = acc;
  }
}

// Validates the key ranges: 0 <= kb[u] <= ke[u] <= n_keys (else SA_ERR_BAD_OFFSETS).
__global__ void check_ranges_kernel(const int64_t* __restrict__ kb, const int64_t* __restrict__ ke,
                                    int R, long long n_keys, WsHeader* hdr) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < R; u += gridDim.x * blockDim.x)
    if (kb[u] < 0 || ke[u] < kb[u] || ke[u] > n_keys) latch_status(&hdr->status, SA_ERR_BAD_OFFSETS);
}

// The recent branch's keys: user u's last min(n_u, L) history rows.
__global__ void recent_ranges_kernel(const int64_t* __restrict__ off, int R, long long L,
                                     int64_t* __restrict__ kb, int64_t* __restrict__ ke) {
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < R; u += gridDim.x * blockDim.x) {
    const long long a = off[u], b = off[u + 1];
    kb[u] = b - a > L ? b - L : a;
    ke[u] = b;
  }
}


GemmOperandDesc opk(const void* base, uint64_t rows, uint64_t cols, bool mn_major) {
  GemmOperandDesc o;
  o.base = base;
  o.rows = rows;
  o.cols = cols;
  o.mn_major = mn_major;
  return o;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// Steps shared by the forward and the backward: schedule, range check, Q', and the flash
// kernel (O' [n_cand, d] fp32 and lse2 into the workspace; lse if asked).
cudaError_t keys_core(const StcaKeysArgs& a, float* lse, bool fwd_call, cudaStream_t s) {
  const StcaKeysPlan& p = a.plan;
  WsHeader* hdr = at<WsHeader>(a.workspace, p.hdr);
  long long* ts = at<long long>(a.workspace, p.ts);
  cudaError_t e;
  if ((e = launch_schedule(a.coff, a.R, a.n_cand, hdr, ts, s)) != cudaSuccess) return e;
  if (a.R > 0) {
    check_ranges_kernel<<<(a.R + 255) / 256, 256, 0, s>>>(a.kb, a.ke, a.R, a.n_keys, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const long long n = a.n_cand;
  const int d = a.d;
  if (n == 0) return cudaSuccess;
  float* O = at<float>(a.workspace, p.o);
  float* lse2 = at<float>(a.workspace, p.lse2);
  if (a.n_keys == 0) {
    keys_empty_kernel<<<1024, 256, 0, s>>>(n, d, O, lse2, lse);
    return cudaGetLastError();
  }
  // M = W_q W_K^T (fp32), then Q' = Q M log2(e) / sqrt(d) in fp32, stored as bf16 hi + lo
  float* M = at<float>(a.workspace, p.mt);
  __nv_bfloat16* Qh = at<__nv_bfloat16>(a.workspace, p.qh);
  __nv_bfloat16* Ql = at<__nv_bfloat16>(a.workspace, p.ql);
  const float qscale = kLog2e / std::sqrt((float)d);
  if ((e = d == 64 ? launch_folds<64>(a.Wq, a.WK, a.Q, n, qscale, M, Qh, Ql, s)
                   : launch_folds<128>(a.Wq, a.WK, a.Q, n, qscale, M, Qh, Ql, s)) != cudaSuccess)
    return e;
  CUtensorMap tqh, tql, tk;
  if (!tmap_rows_bf16(&tqh, Qh, (uint64_t)n, d) || !tmap_rows_bf16(&tql, Ql, (uint64_t)n, d) ||
      !tmap_rows_bf16(&tk, a.Kx, (uint64_t)a.n_keys, d))
    return cudaErrorInvalidValue;
  const long long grid = n / 128 + a.R + 1;  // bounds the candidate tiles; the rest exit
  if (fwd_call && (e = prof_mark_start(s)) != cudaSuccess) return e;
  if (d == 64) {
    const size_t smem = 1024 + KSmem<64>::oBars + sizeof(KBars);
    if ((e = cudaFuncSetAttribute(stca_keys_fwd_kernel<64>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    stca_keys_fwd_kernel<64><<<(unsigned)grid, kThreads, smem, s>>>(
        tqh, tql, tk, a.coff, a.kb, a.ke, a.R, hdr, ts, O, lse2, lse, kDefaultWaitBudget);
  } else {
    const size_t smem = 1024 + KSmem<128>::oBars + sizeof(KBars);
    if ((e = cudaFuncSetAttribute(stca_keys_fwd_kernel<128>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    stca_keys_fwd_kernel<128><<<(unsigned)grid, kThreads, smem, s>>>(
        tqh, tql, tk, a.coff, a.kb, a.ke, a.R, hdr, ts, O, lse2, lse, kDefaultWaitBudget);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return fwd_call ? prof_mark_stop(s) : cudaSuccess;
}

}  // namespace

// 2-D tensor map over bf16 rows [rows, cols]: boxes of 64 columns x 128 rows, 128B swizzle.
bool tmap_rows_bf16(CUtensorMap* m, const void* base, uint64_t rows, int cols) {
  auto fn = tmap_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t stca_keys_plan(int R, long long n_cand, int d, bool backward, int sms, StcaKeysPlan* p) {
  StcaKeysPlan q;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at_ = o;
    o = (o + bytes + 255) / 256 * 256;
    return at_;
  };
  const size_t n = (size_t)n_cand, nd = n * d;
  q.hdr = take(sizeof(WsHeader));
  q.ts = take((size_t)(R + 1) * sizeof(long long));
  q.mt = take((size_t)d * d * sizeof(float));
  q.qh = take(nd * 2);
  q.ql = take(nd * 2);
  q.o = take(nd * sizeof(float));
  q.lse2 = take(n * sizeof(float));
  q.ohi = take(nd * 2);
  q.olo = take(nd * 2);
  if (backward) {
    const long long kt = ((long long)n + 63) / 64;
    long long sp = 2LL * (sms > 0 ? sms : 148);
    if (sp > kt) sp = kt;
    q.splits = (int)(sp < 1 ? 1 : sp);
    q.mts = take((size_t)d * d * 2);
    q.ghi = take(nd * 2);
    q.glo = take(nd * 2);
    q.gb = take(nd * 2);
    q.do_f = take(nd * sizeof(float));
    q.do_b = take(nd * 2);
    q.ob = take(nd * 2);
    q.dd = take(n * sizeof(float));
    q.g1 = take(nd * sizeof(float));
    q.g1hi = take(nd * 2);
    q.g1lo = take(nd * 2);
    q.part = take((size_t)q.splits * d * d * sizeof(float));
    q.dm = take((size_t)d * d * sizeof(float));
  }
  q.total = o;
  *p = q;
  return o;
}

cudaError_t launch_stca_keys_forward(const StcaKeysArgs& a, cudaStream_t s) {
  const StcaKeysPlan& p = a.plan;
  cudaError_t e;
  if ((e = keys_core(a, a.lse, true, s)) != cudaSuccess) return e;
  const long long n = a.n_cand;
  if (n == 0) return cudaSuccess;
  const int d = a.d;
  const WsHeader* hdr = at<WsHeader>(a.workspace, p.hdr);
  __nv_bfloat16* hi = at<__nv_bfloat16>(a.workspace, p.ohi);
  __nv_bfloat16* lo = at<__nv_bfloat16>(a.workspace, p.olo);
  if ((e = stca_split_hilo(at<float>(a.workspace, p.o), n * d, hi, lo, s)) != cudaSuccess) return e;
  // out = (hi + lo) W_V, W_V[f][e]: rows = K, cols = N
  return gemm_hilo(hdr, hi, lo, n, d, opk(a.WV, (uint64_t)d, (uint64_t)d, true), a.out, s);
}

cudaError_t launch_stca_keys_backward(const StcaKeysArgs& a, const StcaKeysGrads& gr,
                                      cudaStream_t s) {
  const StcaKeysPlan& p = a.plan;
  void* ws = a.workspace;
  auto bf = [&](size_t off) { return at<__nv_bfloat16>(ws, off); };
  auto f32 = [&](size_t off) { return at<float>(ws, off); };
  const WsHeader* hdr = at<WsHeader>(ws, p.hdr);
  const int R = a.R, d = a.d;
  const long long n = a.n_cand;
  const float isd = 1.0f / std::sqrt((float)d);
  cudaError_t e;
  if ((e = keys_core(a, nullptr, false, s)) != cudaSuccess) return e;
  if (a.n_keys > 0 && !gr.accumulate &&
      (e = cudaMemsetAsync(gr.dKx, 0, (size_t)a.n_keys * d * sizeof(float), s)) != cudaSuccess)
    return e;
  if (n == 0) {
    for (float* g : {gr.dWq, gr.dWK, gr.dWV})
      if ((e = cudaMemsetAsync(g, 0, (size_t)d * d * sizeof(float), s)) != cudaSuccess) return e;
    return cudaSuccess;
  }
  const float* O = f32(p.o);
  // G = dL/dout as hi + lo (for dO') and bf16 (for dW_V); O' as bf16 (for dW_V)
  if ((e = stca_split_hilo(gr.dout, n * d, bf(p.ghi), bf(p.glo), s)) != cudaSuccess) return e;
  if ((e = stca_to_bf16(gr.dout, n * d, bf(p.gb), s)) != cudaSuccess) return e;
  if ((e = stca_to_bf16(O, n * d, bf(p.ob), s)) != cudaSuccess) return e;
  // dO' = G W_V^T: B[n = f][k = e] = W_V[f][e], K-major
  if ((e = gemm_hilo(hdr, bf(p.ghi), bf(p.glo), n, d, opk(a.WV, (uint64_t)d, (uint64_t)d, false),
                     f32(p.do_f), s)) != cudaSuccess)
    return e;
  // dW_V = O'^T G
  if ((e = gemm_tn_sum(hdr, bf(p.ob), bf(p.gb), n, d, p.splits, f32(p.part), 1.0f, gr.dWV, s)) !=
      cudaSuccess)
    return e;
  // dO' in bf16 (the MMAs' operand) and D_c = bf16(dO'_c) . O'_c, consistent with it
  if ((e = stca_to_bf16(f32(p.do_f), n * d, bf(p.do_b), s)) != cudaSuccess) return e;
  keys_rowdot_kernel<<<1024, 256, 0, s>>>(bf(p.do_b), O, n, d, f32(p.dd));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.n_keys > 0) {  // G1 and dKx on the tensor cores
    StcaKeysBwdArgs k;
    k.Qh = bf(p.qh);
    k.Ql = bf(p.ql);
    k.dOb = bf(p.do_b);
    k.Kx = a.Kx;
    k.n_keys = a.n_keys;
    k.n_cand = n;
    k.coff = a.coff;
    k.kb = a.kb;
    k.ke = a.ke;
    k.R = R;
    k.d = d;
    k.hdr = hdr;
    k.tile_start = at<long long>(ws, p.ts);
    k.lse2 = f32(p.lse2);
    k.Dd = f32(p.dd);
    k.G1 = f32(p.g1);
    k.dKx = gr.dKx;
    if ((e = prof_mark_start(s)) != cudaSuccess) return e;
    if ((e = launch_stca_keys_bwd_kernel(k, s)) != cudaSuccess) return e;
    if ((e = prof_mark_stop(s)) != cudaSuccess) return e;
  } else if ((e = cudaMemsetAsync(f32(p.g1), 0, (size_t)n * d * sizeof(float), s)) != cudaSuccess) {
    return e;
  }
  // dQ = G1 M^T / sqrt(d) (Mts = M^T / sqrt(d) stored [f][r]: B MN-major, rows = K = f)
  if ((e = stca_split_hilo(f32(p.g1), n * d, bf(p.g1hi), bf(p.g1lo), s)) != cudaSuccess) return e;
  if ((e = launch_fold(a.WK, a.Wq, SA_BF16, d, d, d, isd, bf(p.mts), true, s)) != cudaSuccess)
    return e;
  if ((e = gemm_hilo(hdr, bf(p.g1hi), bf(p.g1lo), n, d, opk(bf(p.mts), (uint64_t)d, (uint64_t)d, true),
                     gr.dQ, s)) != cudaSuccess)
    return e;
  // dM = Q^T G1 / sqrt(d), then dW_q = dM W_K and dW_K = dM^T W_q
  if ((e = stca_to_bf16(f32(p.g1), n * d, bf(p.gb), s)) != cudaSuccess) return e;
  if ((e = gemm_tn_sum(hdr, static_cast<const __nv_bfloat16*>(a.Q), bf(p.gb), n, d, p.splits,
                       f32(p.part), isd, f32(p.dm), s)) != cudaSuccess)
    return e;
  return stca_weight_grads(f32(p.dm), a.Wq, a.WK, d, gr.dWq, gr.dWK, s);
}

cudaError_t launch_recent_ranges(const int64_t* offsets, int R, int64_t L, int64_t* kb,
                                 int64_t* ke, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  recent_ranges_kernel<<<(R + 255) / 256, 256, 0, s>>>(offsets, R, L, kb, ke);
  return cudaGetLastError();
}

}  // namespace sa
