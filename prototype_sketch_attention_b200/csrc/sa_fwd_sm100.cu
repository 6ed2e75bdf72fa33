// Sketch Attention forward on tcgen05 tensor cores (sm_100a), bf16 in / fp32 accumulate.
//
// What is computed (blog "100,000 videos in your pocket", section "1. Sketch Attention
// compresses the history"; evolve.pub review "Summary"): for every history token the k
// prototypes' scores are normalised ACROSS PROTOTYPES (each token spreads unit mass),
// and each prototype accumulates the mass-weighted sum of tokens. The projections are
// folded away before this kernel: with P' = P W_k^T log2(e)/sqrt(d) (bf16, computed by
// the fold kernel), the score of prototype j on token t in log2 units is P'_j . X_t, and
// sum_t A_jt V_t = (sum_t A_jt X_t) W_v, applied later in the finalize kernel.
//
// Decomposition. A cluster of C = ceil(k/128) CTAs owns one slice of the token stream; CTA
// of rank c owns prototypes [128c, 128c+128). Per tile of 128 tokens each CTA:
//   1. TMA loads the X tile (128 x d bf16, 128B swizzle, 64-column boxes) into one of NS
//      shared-memory stages; the stages share one all-ones atom (see FwdSmem).
//      Every CTA loads the tile itself (no multicast; the C-fold re-read is served by L2,
//      and rank 0 prefetches upcoming tiles into L2).
//   2. tcgen05.mma  S^T[tok, proto] = X_tile . P'_slice^T  into TMEM (fp32, two
//      buffers), so a token's scores sit in one TMEM lane and one thread owns one token.
//   3. Two softmax warpgroups take alternate tiles. Each thread loads its token's row,
//      takes the local max m and l = m + log2 sum 2^(s - m), and sends l to every CTA of
//      the cluster with st.async (DSMEM); once all C partials are in,
//      lse2 = log2 sum_c 2^(l_c) and A = 2^(s - lse2).
//   4. A is written as bf16 into shared memory in the MN-major layout of the next MMA's
//      A operand, then  [U | mass] += A . [X_tile | 1]  (one tcgen05.mma with N = d + 16,
//      accumulator in TMEM): the 16 extra columns read the all-ones atom and carry the
//      per-prototype mass sum_t A_jt.
//   5. When the token stream crosses a user boundary (or the slice ends) the partial
//      (U, mass) of that (cluster, user) segment is written to the workspace; the finalize
//      kernel adds the segments of each user in a fixed order (deterministic).
// Roles: warp 0 TMA producer, warp 1 allocates TMEM and issues the score MMAs, warp 2 the
// accumulate MMAs, warp 3 idle, warps 4-11 the softmax warpgroups. All mbarrier waits are
// bounded (see sa_common.cuh).
#include <cuda.h>

#include <cmath>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kProtoSlice = 128;              // prototypes per CTA (TMEM lanes / MMA M)
constexpr int kMaxCluster = SA_MAX_K / kProtoSlice;  // CTAs per cluster at most
constexpr int kXchSlots = 4;                  // exchange slots (tile index mod 4)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColU = 256;

// Shared memory in 16 KB slots (one 128-row x 128-byte swizzled atom column each).
//
// X arrives in boxes of 64 columns with the 128-byte swizzle (a 32 KB tile moves in
// two TMA boxes; measured on B200, that lands in under half the time of eight 16-column
// boxes). MMA2 reads [X | 1] as one MN-major operand of width d + 16: its 64-column
// atoms sit LBO bytes apart and the all-ones block is the atom after the last X atom.
// The descriptor's LBO is per stage, so every stage can end on ONE shared ones atom:
// stage s puts X box b at slot kOnes - (d/64 - b) * a_s and uses LBO = a_s slots, with
// the a_s chosen so that no two stages share a slot (d = 128: a = 1, 3, 4, 5 -> slots
// {8,9}, {4,7}, {2,6}, {0,5}; the free slots 1 and 3 hold the A tile).
//
// The A tile is single-buffered at d = 128 (NA = 1), and the slots that frees buy a
// fourth X stage (an X stage is held from its load through the scores, the softmax and
// the accumulate MMA). One A buffer makes "A(i) store -> MMA2(i) -> A(i+1) store" a
// chain on every tile; the softmax computes A in registers before it waits for the
// buffer, and score MMAs are held back so that MMA2 does not queue behind them
// (kMma1Lead), which keeps that chain below the softmax's own per-tile time.
template <int D, int NS, int NA>
struct FwdSmem {
  static constexpr int kSlot = 16384;
  static constexpr int kXBoxes = D / 64;
  static constexpr int kXBytes = 128 * D * 2;                // X tile
  static constexpr int kPBytes = kProtoSlice * D * 2;        // P' slice
  static_assert((D == 128 && NA == 1 && (NS == 4 || NS == 3)) || (D == 64 && NS == 4 && NA == 2),
                "layout");
  static constexpr int kOnes = D == 128 ? (NS == 4 ? 10 : 8) : 4;
  // stage spacing a_s (in slots): d = 128: 1, 3, 4, 5; d = 64: 1, 2, 3, 4
  __host__ __device__ static constexpr int stage_a(int s) {
    return D == 128 ? (s == 0 ? 1 : s == 1 ? 3 : s == 2 ? 4 : 5) : s + 1;
  }
  // byte offset of X box b of stage s; of the A buffer's two 64-prototype atoms
  __host__ __device__ static constexpr int xbox(int s, int b) {
    return (kOnes - (kXBoxes - b) * stage_a(s)) * kSlot;
  }
  __host__ __device__ static constexpr int abox(int buf, int mb) {
    return (D == 128 ? (NS == 4 ? (mb == 0 ? 1 : 3) : (mb == 0 ? 1 : 3))
                     : (buf == 0 ? (mb == 0 ? 5 : 6) : (mb == 0 ? 7 : 8))) * kSlot;
  }
  static constexpr int oOnes = kOnes * kSlot;
  static constexpr int oP = (D == 128 ? (NS == 4 ? 11 : 9) : 9) * kSlot;
  static constexpr int oXch = oP + kPBytes;  // kXchSlots * C * 128 floats (runtime C)
  static size_t bytes(int C) {
    const size_t xch = (size_t)kXchSlots * C * 128 * 4;
    const size_t bars = 64 * 8 + 16;
    return 1024 + oXch + xch + bars;
  }
};

struct Bars {
  uint64_t x_full[4], x_empty[4];
  uint64_t s_full[2], s_empty[2];
  uint64_t a_full[2], a_empty[4];
  uint64_t u_full[2], u_empty;  // u_full[w]: segments whose last tile warpgroup w owns
  uint64_t xch[kXchSlots];
  uint64_t p_full, drain, drain2;
  uint64_t m2iss[4];  // MMA2(i) issued, by tile mod 4 (orders MMA1 behind it)
  uint32_t tmem_base;
};

__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr) : "memory");
  return __uint_as_float(r);
}

constexpr int kNWG = 2;                        // softmax warpgroups (ping-pong on tiles)
// warps 0-3: TMA producer (0), TMEM allocator and MMA1 issuer (1), MMA2 issuer (2),
// idle (3); warps 4-11: the two softmax warpgroups
constexpr int kThreads = 128 + 128 * kNWG;
constexpr int kPrefetchAhead = 4;               // tiles prefetched into L2 ahead of the load
// MMA1(i) is issued only after MMA2(i - kMma1Lead). The tensor pipe runs its queue in
// order, and an accumulate MMA queued behind a score MMA waits for it; the accumulate MMA
// is on the chain "A store -> MMA2 -> next A store" (one A buffer), while the score MMA of
// tile i is needed only when its warpgroup finishes tile i - 2. With a lead of 3 the score
// MMAs fill the gaps instead.
constexpr int kMma1Lead = 3;

// Scores of this thread's token (one TMEM lane) for the CTA's 128 prototypes.
__device__ __forceinline__ void load_scores(uint32_t taddr, float (&v)[kProtoSlice]) {
  uint32_t r0[32], r1[32], r2[32], r3[32];
  tmem_ld32_raw(taddr + 0, r0);
  tmem_ld32_raw(taddr + 32, r1);
  tmem_ld32_raw(taddr + 64, r2);
  tmem_ld32_raw(taddr + 96, r3);
  tmem_wait_tie(r0);
  tmem_wait_tie(r1);
  tmem_wait_tie(r2);
  tmem_wait_tie(r3);
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    v[x] = __uint_as_float(r0[x]);
    v[32 + x] = __uint_as_float(r1[x]);
    v[64 + x] = __uint_as_float(r2[x]);
    v[96 + x] = __uint_as_float(r3[x]);
  }
}

// v <- 2^v in place; returns the sum (four packed accumulators, then a tree).
__device__ __forceinline__ float exp2_and_sum(float (&v)[kProtoSlice]) {
  uint64_t za[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int p = 0; p < kProtoSlice / 2; ++p) {
    v[2 * p] = ex2_approx(v[2 * p]);
    v[2 * p + 1] = ex2_approx(v[2 * p + 1]);
    za[p & 3] = f2_add(za[p & 3], f2_pack(v[2 * p], v[2 * p + 1]));
  }
  float z0, z1;
  f2_unpack(f2_add(f2_add(za[0], za[1]), f2_add(za[2], za[3])), z0, z1);
  return z0 + z1;
}

// sum over the 128 scores of 2^(v - m), v left unchanged (four packed accumulators).
__device__ __forceinline__ float sum_exp2(const float (&v)[kProtoSlice], float m) {
  uint64_t za[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int p = 0; p < kProtoSlice / 2; ++p)
    za[p & 3] = f2_add(za[p & 3], f2_pack(ex2_approx(v[2 * p] - m), ex2_approx(v[2 * p + 1] - m)));
  float z0, z1;
  f2_unpack(f2_add(f2_add(za[0], za[1]), f2_add(za[2], za[3])), z0, z1);
  return z0 + z1;
}

// Maximum of the 128 scores: four independent chains of 3-input max.
__device__ __forceinline__ float row_max(const float (&v)[kProtoSlice]) {
  float mc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float a = fmaxf(v[32 * j], v[32 * j + 31]);
#pragma unroll
    for (int c = 1; c < 31; c += 2) a = fmax3(a, v[32 * j + c], v[32 * j + c + 1]);
    mc[j] = a;
  }
  return fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
}

// One 64-prototype block of token row r into the MN-major, 128B-swizzled A operand.
__device__ __forceinline__ void store_a_block(uint8_t* arow, int r, const uint32_t (&a)[32]) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    *reinterpret_cast<uint4*>(arow + ((ch ^ (r & 7)) << 4)) =
        make_uint4(a[ch * 4], a[ch * 4 + 1], a[ch * 4 + 2], a[ch * 4 + 3]);
}

// log2 of the sum of 2^x[p * 128] over the C partials of one token (C <= MAXC).
// Every load and exponential is independent; max and sum are trees. MAXC is the
// kernel's cluster-size bound, which keeps the register footprint at MAXC.
template <int MAXC>
__device__ __forceinline__ float combine_partials(const float* x, int C) {
  float lp[MAXC], t[MAXC];
#pragma unroll
  for (int p = 0; p < MAXC; ++p) lp[p] = p < C ? x[p * 128] : -INFINITY;
#pragma unroll
  for (int p = 0; p < MAXC; ++p) t[p] = lp[p];
#pragma unroll
  for (int w = MAXC / 2; w >= 1; w /= 2)
#pragma unroll
    for (int p = 0; p < w; ++p) t[p] = fmaxf(t[p], t[p + w]);
  const float mx = t[0];
#pragma unroll
  for (int p = 0; p < MAXC; ++p) t[p] = p < C ? ex2_approx(lp[p] - mx) : 0.f;
#pragma unroll
  for (int w = MAXC / 2; w >= 1; w /= 2)
#pragma unroll
    for (int p = 0; p < w; ++p) t[p] += t[p + w];
  return mx + lg2_approx(t[0]);
}

template <int D, int NS, int NA>
__global__ void __launch_bounds__(kThreads, 1)
sa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_p,
                    const int64_t* __restrict__ offsets, int R, int k_valid, int C, int k_pad,
                    WsHeader* hdr, const long long* __restrict__ tile_start,
                    float* __restrict__ part_u, float* __restrict__ part_m,
                    float* __restrict__ lse_out, int H, int share, long long budget) {
  using L = FwdSmem<D, NS, NA>;
  constexpr int KSTEPS1 = D / 16;           // MMA1 K steps (over d)
  constexpr int KSTEPS2 = kTileTokens / 16;  // MMA2 K steps (over tokens)
  constexpr int kMaxC = (D == 128 && NS == 4) ? 8 : kMaxCluster;  // cluster-size bound
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* xch = reinterpret_cast<float*>(smem + L::oXch);
  Bars* bars = reinterpret_cast<Bars*>(smem + L::oXch + (size_t)kXchSlots * C * 128 * 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t cid = cluster_id_x(), ncl = nclusters_x();
  int* status = &hdr->status;

  // ---- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bars->x_full[s]), 1);
      mbar_init(smem_u32(&bars->x_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->s_full[s]), 1);
      mbar_init(smem_u32(&bars->s_empty[s]), 4);
      mbar_init(smem_u32(&bars->a_full[s]), 4);
      mbar_init(smem_u32(&bars->a_empty[s]), 1);
      mbar_init(smem_u32(&bars->a_empty[s + 2]), 1);
    }
    mbar_init(smem_u32(&bars->u_full[0]), 1);
    mbar_init(smem_u32(&bars->u_full[1]), 1);
    mbar_init(smem_u32(&bars->u_empty), 4);
    for (int s = 0; s < kXchSlots; ++s) mbar_init(smem_u32(&bars->xch[s]), 1);
    mbar_init(smem_u32(&bars->p_full), 1);
    for (int s = 0; s < 4; ++s) mbar_init(smem_u32(&bars->m2iss[s]), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    mbar_init(smem_u32(&bars->drain2), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 4) {
    // the shared all-ones atom read by MMA2 after the X atoms (N = d + 16): its 16 extra
    // output columns accumulate sum_t A_jt (the mass) next to U
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + L::oOnes);
    for (int w = threadIdx.x - 128; w < L::kSlot / 4; w += kThreads - 128) ones[w] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // peers' barriers are initialised before any st.async arrives
  tc_fence_after();
  // every CTA is resident: the helper grid queued behind this one may take the free SMs
  griddep_launch_dependents();
  const uint32_t tmem = bars->tmem_base;

  // this cluster's range of the token tiles
  const long long T = read_status(status) == 0 ? hdr->total_tiles : 0;
  const TileRanges rg(T, (int)ncl, H, share);
  const long long ta = rg.start(cid), tb = rg.start(cid + 1);

  if (warp == 0) {
    // ================= TMA producer (+ L2 prefetch of upcoming tiles by rank 0)
    if (lane == 0 && ta < tb) {
      tma_prefetch_desc(&tmap_x);
      tma_prefetch_desc(&tmap_p);
      const uint32_t pf = smem_u32(&bars->p_full);
      mbar_arrive_expect_tx(pf, L::kPBytes);
      for (int b = 0; b < D / 64; ++b)
        tma_load_2d(sbase + L::oP + b * L::kSlot, &tmap_p, b * 64, (int)rank * kProtoSlice, pf);
      TileIter it, ahead;
      it.init(tile_start, offsets, R, ta, tb);
      ahead.init(tile_start, offsets, R, ta, tb);
      if (rank == 0) {
        for (int j = 0; j < kPrefetchAhead && ahead.valid(); ++j, ahead.next())
          for (int b = 0; b < L::kXBoxes; ++b) tma_prefetch_l2_2d(&tmap_x, b * 64, (int)ahead.t0());
      }
      int i = 0;
      for (; it.valid(); it.next(), ++i) {
        const int st = (int)(i % NS);
        const uint32_t par = (uint32_t)((i / NS) & 1);
        if (!mbar_wait(smem_u32(&bars->x_empty[st]), par ^ 1u, status, budget)) break;
        const uint32_t fb = smem_u32(&bars->x_full[st]);
        mbar_arrive_expect_tx(fb, L::kXBytes);
        const int y = (int)it.t0();
        for (int b = 0; b < L::kXBoxes; ++b)
          tma_load_2d(sbase + L::xbox(st, b), &tmap_x, b * 64, y, fb);
        if (rank == 0 && ahead.valid()) {
          for (int b = 0; b < L::kXBoxes; ++b) tma_prefetch_l2_2d(&tmap_x, b * 64, (int)ahead.t0());
          ahead.next();
        }
      }
      // drain: the loads of the last NS tiles issued must have landed before exit
      for (long long j = (i > NS ? i - NS : 0); j < i; ++j)
        mbar_wait_drain(smem_u32(&bars->x_full[j % NS]), (uint32_t)((j / NS) & 1), budget);
      mbar_wait_drain(pf, 0, budget);
    }
  } else if (warp == 1 || warp == 2) {
    // ================= MMA issuers: warp 1 issues MMA1 (scores), warp 2 MMA2 (accumulate)
    if (lane == 0 && ta < tb) {
      const uint32_t idesc1 = idesc_bf16_f32(128, kProtoSlice, 0, 0);
      const uint32_t idesc2 = idesc_bf16_f32(128, D + 16, 1, 1);
      // Shared-memory descriptors built once per operand base; a later operand address is
      // the same descriptor plus (byte offset >> 4) in its 14-bit address field (every
      // operand lies below 256 KB, so the field never carries).
      const uint64_t dp1 = smem_desc(sbase + L::oP, 16, 1024, kSwizzle128B);  // P', K-major
      const uint64_t da2_0 =                                                  // A, MN-major
          smem_desc(sbase + L::abox(0, 0), L::abox(0, 1) - L::abox(0, 0), 1024, kSwizzle128B);
      const uint64_t da2_1 =
          smem_desc(sbase + L::abox(1, 0), L::abox(1, 1) - L::abox(1, 0), 1024, kSwizzle128B);
      bool ok = mbar_wait(smem_u32(&bars->p_full), 0, status, budget);
      TileIter it;
      it.init(tile_start, offsets, R, ta, tb);
      int i = 0;
      int seg = -1, prev_u = -1;
      for (; ok && it.valid(); it.next(), ++i) {
        const bool first = it.u != prev_u, last = it.last();  // first tile of a segment
        prev_u = it.u;
        if (first) ++seg;
        const int st = (int)(i % NS);
        const int sb = (int)(i & 1);
        if (warp == 1) {
          // m2iss[(i - kMma1Lead) mod 4]: MMA1(i - 4) already waited for MMA2(i - 4 - kMma1Lead),
          // so only that phase or the awaited one are possible (one parity bit)
          ok = mbar_wait(smem_u32(&bars->x_full[st]), (uint32_t)((i / NS) & 1), status, budget) &&
               mbar_wait(smem_u32(&bars->s_empty[sb]), (uint32_t)(((i >> 1) & 1) ^ 1), status, budget) &&
               (i < kMma1Lead ||
                mbar_wait(smem_u32(&bars->m2iss[(i - kMma1Lead) & 3]),
                          (uint32_t)(((i - kMma1Lead) >> 2) & 1), status, budget));
          if (!ok) break;
          tc_fence_after();
          // A = X tile, K-major, 128B swizzle: four 16-wide K steps per 64-column box
          uint64_t xd[L::kXBoxes];
#pragma unroll
          for (int b = 0; b < L::kXBoxes; ++b)
            xd[b] = smem_desc(sbase + L::xbox(st, b), 16, 1024, kSwizzle128B);
#pragma unroll
          for (int ks = 0; ks < KSTEPS1; ++ks) {
            const uint32_t koff = (ks >> 2) * L::kSlot + (ks & 3) * 32;
            tc_mma_f16(tmem + (sb ? kColS1 : kColS0), xd[ks >> 2] + (uint64_t)(((ks & 3) * 32) >> 4),
                       dp1 + (uint64_t)(koff >> 4), idesc1, ks > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars->s_full[sb]));
        } else {
          const int ab = NA == 2 ? sb : 0;
          const uint32_t apar = NA == 2 ? (uint32_t)((i >> 1) & 1) : (uint32_t)(i & 1);
          ok = mbar_wait(smem_u32(&bars->a_full[ab]), apar, status, budget) &&
               (!first || mbar_wait(smem_u32(&bars->u_empty), (uint32_t)((seg & 1) ^ 1), status, budget));
          if (!ok) break;
          tc_fence_after();
          // A = A tile, MN-major (prototypes contiguous); B = [X | 1], MN-major (d contiguous),
          // its atoms LBO = a_s slots apart ending on the shared ones atom; both 128B swizzle,
          // a 16-token K step is two 8-row groups (2048 bytes)
          const uint64_t ad0 = ab ? da2_1 : da2_0;
          const uint64_t xd = smem_desc(sbase + L::xbox(st, 0), L::stage_a(st) * L::kSlot, 1024,
                                        kSwizzle128B);
#pragma unroll
          for (int ks = 0; ks < KSTEPS2; ++ks)
            tc_mma_f16(tmem + kColU, ad0 + (uint64_t)((ks * 2048) >> 4), xd + (uint64_t)((ks * 2048) >> 4),
                       idesc2, (first && ks == 0) ? 0u : 1u);
          tc_commit(smem_u32(&bars->x_empty[st]));
          // with one A buffer, a_empty is indexed by tile mod 4 (see the A store)
          tc_commit(smem_u32(&bars->a_empty[NA == 2 ? ab : (i & 3)]));
          if (last) tc_commit(smem_u32(&bars->u_full[i & 1]));
          mbar_arrive(smem_u32(&bars->m2iss[i & 3]));  // lets MMA1(i + kMma1Lead) in
        }
      }
      const uint32_t db = smem_u32(warp == 1 ? &bars->drain : &bars->drain2);
      tc_commit(db);
      mbar_wait_drain(db, 0, budget);
    }
  } else if (warp >= 4) {
    // ================= softmax + epilogue: warpgroup wg takes the tiles i with i % 2 == wg
    const int wg = (warp >> 2) - 1;
    const int q = warp & 3;                   // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;              // token row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool leader = (threadIdx.x & 127) == 0;
    const int pbase = (int)rank * kProtoSlice;
    const bool partial_slice = pbase + kProtoSlice > k_valid;
    TileIter it;
    it.init(tile_start, offsets, R, ta, tb);
    int i = 0;
    int useg = 0;  // segments whose last tile this warpgroup owned so far (u_full[wg] phases)
    bool ok = true;
    for (; ok && it.valid(); it.next(), ++i) {
      if ((int)(i & 1) != wg) continue;
      const int sb = wg;
      if (!mbar_wait_warp(smem_u32(&bars->s_full[sb]), (uint32_t)((i >> 1) & 1), status, budget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_tmem = tmem + lane_off + (sb ? kColS1 : kColS0);
      float v[kProtoSlice];
      load_scores(s_tmem, v);
      if (partial_slice) {
#pragma unroll
        for (int c = 0; c < kProtoSlice; ++c)
          if (pbase + c >= k_valid) v[c] = -INFINITY;
      }
      // e = 2^s and z = sum e without a max shift: exact whenever z stays within
      // [2^-100, 2^100], which holds unless a token's scores are extreme. A warp with
      // any lane outside that range reloads its scores and takes the shifted path.
      float m = 0.f;
      float z = exp2_and_sum(v);
      const bool in_range = z >= 0x1p-100f && z <= 0x1p100f;
      if (!__all_sync(0xffffffffu, in_range)) {
        load_scores(s_tmem, v);
        if (partial_slice) {
#pragma unroll
          for (int c = 0; c < kProtoSlice; ++c)
            if (pbase + c >= k_valid) v[c] = -INFINITY;
        }
        m = row_max(v);
#pragma unroll
        for (int c = 0; c < kProtoSlice; ++c) v[c] -= m;
        z = exp2_and_sum(v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty[sb]));
      const int nv = it.nvalid();
      const bool valid = r < nv;
      const float l = valid ? m + lg2_approx(z) : 0.f;

      // exchange l with every CTA of the cluster (4 tokens per 16-byte st.async)
      const int qs = (int)(i & (kXchSlots - 1));
      const uint32_t xbar = smem_u32(&bars->xch[qs]);
      {
        const int g0 = lane & ~3;
        const float v0 = __shfl_sync(0xffffffffu, l, g0 + 0);
        const float v1 = __shfl_sync(0xffffffffu, l, g0 + 1);
        const float v2 = __shfl_sync(0xffffffffu, l, g0 + 2);
        const float v3 = __shfl_sync(0xffffffffu, l, g0 + 3);
        const uint32_t laddr = smem_u32(xch + ((qs * C + (int)rank) * 128 + q * 32 + g0));
        for (int p = lane & 3; p < C; p += 4)
          st_async_v4(mapa(laddr, (uint32_t)p), v0, v1, v2, v3, mapa(xbar, (uint32_t)p));
      }
      if (leader) mbar_arrive_expect_tx(xbar, (uint32_t)C * 128u * 4u);
      if (!mbar_wait_warp<true>(xbar, (uint32_t)((i >> 2) & 1), status, budget)) {
        ok = false;
        break;
      }
      // lse over the C partials: all loads and exponentials independent (tree reductions)
      const float lse2 = combine_partials<kMaxC>(xch + qs * C * 128 + r, C);
      const float scale = valid ? ex2_approx(m - lse2) : 0.f;
      if (rank == 0 && valid && lse_out != nullptr)
        lse_out[it.t0() + r] = lse2 * 0.69314718055994530942f;

      // A = e * 2^(m - lse2) as bf16 pairs, in registers before the buffer is known free
      // (the wait below is on the chain A store -> MMA2 -> next A store)
      uint32_t pa0[32], pa1[32];
      {
        const uint64_t sc2 = f2_pack(scale, scale);
#pragma unroll
        for (int p = 0; p < 32; ++p) {
          float a, b;
          f2_unpack(f2_mul(f2_pack(v[2 * p], v[2 * p + 1]), sc2), a, b);
          pa0[p] = cvt_bf16x2(a, b);
          f2_unpack(f2_mul(f2_pack(v[64 + 2 * p], v[64 + 2 * p + 1]), sc2), a, b);
          pa1[p] = cvt_bf16x2(a, b);
        }
      }
      // A(i) may overwrite the buffer once MMA2 has read the one before it: with two
      // buffers A(i - 2) (the barrier of this parity), with one A(i - 1) (barrier
      // (i - 1) mod 4, its phase (i - 1) / 4). exp(i) has already seen MMA2(i - NS) complete
      // (its X stage was free), so on either barrier only the awaited phase and the one
      // before it are possible, and one parity bit tells them apart.
      const int ab = NA == 2 ? wg : 0;
      const int eb = NA == 2 ? wg : ((i - 1) & 3);
      const uint32_t epar =
          NA == 2 ? (uint32_t)(((i >> 1) & 1) ^ 1) : (uint32_t)(((i - 1) >> 2) & 1);
      if (!mbar_wait_warp(smem_u32(&bars->a_empty[eb]), epar, status, budget)) {
        ok = false;
        break;
      }
      // A (bf16) into the MN-major, 128B-swizzled A operand: row = token, 64 prototypes
      // per 128-byte row, two 16 KB blocks for prototypes [0,64) and [64,128).
      store_a_block(smem + L::abox(ab, 0) + r * 128, r, pa0);
      store_a_block(smem + L::abox(ab, 1) + r * 128, r, pa1);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->a_full[ab]));

      if (it.last()) {
        // ---- epilogue: this segment's partial (U, mass) for our 128 prototypes
        if (!mbar_wait_warp(smem_u32(&bars->u_full[wg]), (uint32_t)(useg & 1), status, budget)) {
          ok = false;
          break;
        }
        ++useg;
        tc_fence_after();
        const long long sgid = (long long)cid + it.u;
        float* dst = part_u + ((size_t)sgid * k_pad + pbase + r) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u32[32];
          tmem_ld32_raw(tmem + lane_off + kColU + c * 32, u32);
          tmem_wait_tie(u32);
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(dst + c * 32 + x) =
                make_float4(__uint_as_float(u32[x]), __uint_as_float(u32[x + 1]),
                            __uint_as_float(u32[x + 2]), __uint_as_float(u32[x + 3]));
        }
        const float ms = tmem_ld1(tmem + lane_off + kColU + D);
        tc_wait_ld();
        part_m[(size_t)sgid * k_pad + pbase + r] = ms;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->u_empty));
      }
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

// ---------------------------------------------------------------------------- helper CTAs
// Clusters of C CTAs do not tile the SMs exactly (C = 8: 15 clusters on 120 of 148 SMs).
// The SMs left over run helper CTAs, one per SM and without a cluster, on the tail ranges
// of the token tiles (TileRanges: range G + b belongs to helper b). Without a cluster a
// CTA cannot exchange partial log-sums with the CTAs that hold the other prototype slices,
// so a helper does all C slices of its tiles itself, in chunks of kChunk tiles and two
// passes per chunk:
//   pass 1, for each slice s and tile: S = X P'_s^T (MMA1) and the slice's partial
//     l_s = m + log2 sum_j 2^(S_j - m); the token's running lse2 = log2 sum_s 2^(l_s) is
//     kept in shared memory, one float per token;
//   pass 2, for each slice s and tile: S again, A = 2^(S - lse2) and
//     [U_s | mass_s] += A [X | 1] (MMA2) in TMEM; when the slice's pass over the chunk ends,
//     or the tile stream crosses a user boundary, the partial is stored into (first time)
//     or added to the workspace segment (range G + b, user).
// The scores are computed twice, so a helper tile costs about 1.7 to 1.9 times a cluster
// CTA's share of one. The kChunk X tiles of a chunk come from HBM once and from L2 for the
// other 2C - 1 passes.
//
// Ownership rules that make the shared-memory and workspace accesses race-free: tile t of
// a chunk is handled by softmax warpgroup (t & 1) in every pass, so a token's running lse2
// is read and written by one thread only; every segment epilogue is done by warpgroup 0,
// so each workspace row is read and written by one thread only, in program order.
// The score buffers alternate with the tile's parity too, and every role counts each
// buffer's uses itself (chunks may have an odd number of tiles).
constexpr int kChunk = 32;  // tiles per chunk
// Register split: the softmax warpgroups hold a token's 128 scores through both passes'
// sums, so they take 216 registers and the producer / MMA warpgroup gives up all but 64.
// setmaxnreg.inc waits until the block's launch allocation covers it, so the split stays
// within 384 threads x 168 registers, and the launch refuses a build compiled to fewer.
constexpr int kHelperRegsLaunch = 168, kHelperRegsControl = 64, kHelperRegsSoftmax = 216;
static_assert(128 * kHelperRegsControl + 256 * kHelperRegsSoftmax <= kThreads * kHelperRegsLaunch,
              "register split exceeds the launch allocation");

// Shared memory: the clustered kernel's four-stage layout (X stages, A tile, ones atom,
// P' slice), then the running lse2. In pass 2 an X stage is held until the accumulate MMA
// has read it, so the next loads need four stages to hide their L2 latency; that leaves
// room for one P' buffer, which warp 3 reloads between (pass, slice) groups.
template <int D>
struct HelperSmem {
  using X = FwdSmem<D, 4, 1>;
  static constexpr int oL = X::oP + X::kPBytes;  // running lse2, [kChunk][128] floats
  static constexpr int oBars = oL + kChunk * kTileTokens * 4;
};

struct HBars {
  uint64_t x_full[4], x_empty[4];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, p_empty;
  uint64_t a_full, a_empty[4];  // a_empty[i2 mod 4]: MMA2 of pass-2 step i2 has completed
  uint64_t u_full, u_empty;
  uint64_t m2iss[4];
  uint64_t drain, drain2;
  uint32_t tmem_base;
};

template <int D>
constexpr size_t helper_smem_bytes() {
  return 1024 + HelperSmem<D>::oBars + sizeof(HBars);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
sa_fwd_sm100_helper_kernel(const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_p,
                           const int64_t* __restrict__ offsets, int R, int k_valid, int C,
                           int k_pad, WsHeader* hdr, const long long* __restrict__ tile_start,
                           float* __restrict__ part_u, float* __restrict__ part_m,
                           float* __restrict__ lse_out, int G, int H, int share,
                           long long budget) {
  using L = FwdSmem<D, 4, 1>;
  using HS = HelperSmem<D>;
  constexpr int NS = 4;
  constexpr int KSTEPS1 = D / 16;
  constexpr int KSTEPS2 = kTileTokens / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  HBars* bars = reinterpret_cast<HBars*>(smem + HS::oBars);
  float* lsm = reinterpret_cast<float*>(smem + HS::oL);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = &hdr->status;

  // ---- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bars->x_full[s]), 1);
      mbar_init(smem_u32(&bars->x_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->s_full[s]), 1);
      mbar_init(smem_u32(&bars->s_empty[s]), 4);
    }
    mbar_init(smem_u32(&bars->p_full), 1);
    mbar_init(smem_u32(&bars->p_empty), 1);
    mbar_init(smem_u32(&bars->a_full), 4);
    for (int s = 0; s < 4; ++s) {
      mbar_init(smem_u32(&bars->a_empty[s]), 1);
      mbar_init(smem_u32(&bars->m2iss[s]), 1);
    }
    mbar_init(smem_u32(&bars->u_full), 1);
    mbar_init(smem_u32(&bars->u_empty), 4);
    mbar_init(smem_u32(&bars->drain), 1);
    mbar_init(smem_u32(&bars->drain2), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 4) {
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + L::oOnes);
    for (int w = threadIdx.x - 128; w < L::kSlot / 4; w += kThreads - 128) ones[w] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const long long T = read_status(status) == 0 ? hdr->total_tiles : 0;
  const TileRanges rg(T, G, H, share);
  const long long ra = rg.start(G + (long long)blockIdx.x), rb = rg.start(G + (long long)blockIdx.x + 1);

  // each warp changes its register count inside its own role's branch, so that the
  // compiler budgets every role's code for that role's count
  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelperRegsControl));
    // ================= X producer: per step the X tile; the next chunk's tiles are
    // prefetched into L2 during the current chunk's last slice
    if (lane == 0 && ra < rb) {
      tma_prefetch_desc(&tmap_x);
      TileIter base, ahead, it;
      base.init(tile_start, offsets, R, ra, rb);
      ahead = base;
      for (int j = 0; j < kChunk && ahead.valid(); ++j, ahead.next())
        for (int b = 0; b < L::kXBoxes; ++b) tma_prefetch_l2_2d(&tmap_x, b * 64, (int)ahead.t0());
      int i = 0;
      bool ok = true;
      for (long long c0 = ra; ok && c0 < rb; c0 += kChunk) {
        const int K = (int)(rb - c0 < kChunk ? rb - c0 : kChunk);
        for (int ph = 0; ok && ph < 2; ++ph) {
          for (int s = 0; ok && s < C; ++s) {
            const bool track = ph == 0 && s == 0, pref = ph == 1 && s == C - 1;
            if (track) ahead = base;
            it = base;
            for (int tl = 0; tl < K; ++tl, it.next(), ++i) {
              const int st = i % NS;
              if (!mbar_wait(smem_u32(&bars->x_empty[st]), (uint32_t)(((i / NS) & 1) ^ 1), status,
                             budget)) {
                ok = false;
                break;
              }
              const uint32_t fb = smem_u32(&bars->x_full[st]);
              mbar_arrive_expect_tx(fb, L::kXBytes);
              for (int b = 0; b < L::kXBoxes; ++b)
                tma_load_2d(sbase + L::xbox(st, b), &tmap_x, b * 64, (int)it.t0(), fb);
              if (track) {
                ahead.next();
              } else if (pref && ahead.valid()) {
                for (int b = 0; b < L::kXBoxes; ++b)
                  tma_prefetch_l2_2d(&tmap_x, b * 64, (int)ahead.t0());
                ahead.next();
              }
            }
          }
        }
        base = it;
      }
      // drain: the last NS X loads have landed before exit
      for (int j = (i > NS ? i - NS : 0); j < i; ++j)
        mbar_wait_drain(smem_u32(&bars->x_full[j % NS]), (uint32_t)((j / NS) & 1), budget);
    }
  } else if (warp == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelperRegsControl));
    // ================= MMA1 issuer: S[tile parity] = X P'_s^T for every step of both passes.
    // In pass 2, MMA1 of step i2 waits until MMA2(i2 - 3) is issued (so that an accumulate
    // MMA never queues behind a score MMA) and MMA2(i2 - 4) has completed (which bounds how
    // far the A buffer's barriers can lag behind a softmax warpgroup's wait).
    if (lane == 0 && ra < rb) {
      const uint32_t idesc1 = idesc_bf16_f32(128, kProtoSlice, 0, 0);
      const uint64_t dp = smem_desc(sbase + L::oP, 16, 1024, kSwizzle128B);
      int i = 0, q = 0, i2 = 0, nb0 = 0, nb1 = 0;
      bool ok = true;
      for (long long c0 = ra; ok && c0 < rb; c0 += kChunk) {
        const int K = (int)(rb - c0 < kChunk ? rb - c0 : kChunk);
        for (int ph = 0; ok && ph < 2; ++ph) {
          for (int s = 0; ok && s < C; ++s, ++q) {
            if (!mbar_wait(smem_u32(&bars->p_full), (uint32_t)(q & 1), status, budget)) {
              ok = false;
              break;
            }
            for (int tl = 0; tl < K; ++tl, ++i) {
              const int st = i % NS, sb = tl & 1;
              const int nbs = sb ? nb1 : nb0;
              ok = mbar_wait(smem_u32(&bars->x_full[st]), (uint32_t)((i / NS) & 1), status, budget) &&
                   mbar_wait(smem_u32(&bars->s_empty[sb]), (uint32_t)((nbs & 1) ^ 1), status, budget);
              if (ok && ph == 1 && i2 >= 3)
                ok = mbar_wait(smem_u32(&bars->m2iss[(i2 - 3) & 3]), (uint32_t)(((i2 - 3) >> 2) & 1),
                               status, budget);
              if (ok && ph == 1 && i2 >= 4)
                ok = mbar_wait(smem_u32(&bars->a_empty[(i2 - 4) & 3]), (uint32_t)(((i2 - 4) >> 2) & 1),
                               status, budget);
              if (!ok) break;
              tc_fence_after();
              uint64_t xd[L::kXBoxes];
#pragma unroll
              for (int b = 0; b < L::kXBoxes; ++b)
                xd[b] = smem_desc(sbase + L::xbox(st, b), 16, 1024, kSwizzle128B);
#pragma unroll
              for (int ks = 0; ks < KSTEPS1; ++ks) {
                const uint32_t koff = (ks >> 2) * L::kSlot + (ks & 3) * 32;
                tc_mma_f16(tmem + (sb ? kColS1 : kColS0), xd[ks >> 2] + (uint64_t)(((ks & 3) * 32) >> 4),
                           dp + (uint64_t)(koff >> 4), idesc1, ks > 0 ? 1u : 0u);
              }
              tc_commit(smem_u32(&bars->s_full[sb]));
              if (ph == 0) tc_commit(smem_u32(&bars->x_empty[st]));  // pass 1: X is done
              if (tl == K - 1) tc_commit(smem_u32(&bars->p_empty));  // P' slice is done
              if (sb) ++nb1; else ++nb0;
              if (ph == 1) ++i2;
            }
          }
        }
      }
      tc_commit(smem_u32(&bars->drain));
      mbar_wait_drain(smem_u32(&bars->drain), 0, budget);
    }
  } else if (warp == 2) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelperRegsControl));
    // ================= MMA2 issuer (pass 2 only): [U | mass] += A [X | 1]
    if (lane == 0 && ra < rb) {
      const uint32_t idesc2 = idesc_bf16_f32(128, D + 16, 1, 1);
      const uint64_t da =
          smem_desc(sbase + L::abox(0, 0), L::abox(0, 1) - L::abox(0, 0), 1024, kSwizzle128B);
      TileIter base, it;
      base.init(tile_start, offsets, R, ra, rb);
      int i = 0, i2 = 0, seg = 0;
      bool ok = true;
      for (long long c0 = ra; ok && c0 < rb; c0 += kChunk) {
        const int K = (int)(rb - c0 < kChunk ? rb - c0 : kChunk);
        i += C * K;  // pass 1 steps: MMA1 releases their X stages
        for (int s = 0; ok && s < C; ++s) {
          it = base;
          int prev_u = -1;
          for (int tl = 0; tl < K; ++tl, it.next(), ++i, ++i2) {
            const int st = i % NS;
            const bool first = tl == 0 || it.u != prev_u, last = tl == K - 1 || it.last();
            prev_u = it.u;
            ok = mbar_wait(smem_u32(&bars->a_full), (uint32_t)(i2 & 1), status, budget) &&
                 (!first || mbar_wait(smem_u32(&bars->u_empty), (uint32_t)((seg & 1) ^ 1), status, budget));
            if (!ok) break;
            tc_fence_after();
            const uint64_t xd = smem_desc(sbase + L::xbox(st, 0), L::stage_a(st) * L::kSlot, 1024,
                                          kSwizzle128B);
#pragma unroll
            for (int ks = 0; ks < KSTEPS2; ++ks)
              tc_mma_f16(tmem + kColU, da + (uint64_t)((ks * 2048) >> 4), xd + (uint64_t)((ks * 2048) >> 4),
                         idesc2, (first && ks == 0) ? 0u : 1u);
            tc_commit(smem_u32(&bars->x_empty[st]));
            tc_commit(smem_u32(&bars->a_empty[i2 & 3]));
            if (last) {
              tc_commit(smem_u32(&bars->u_full));
              ++seg;
            }
            mbar_arrive(smem_u32(&bars->m2iss[i2 & 3]));
          }
        }
        base = it;
      }
      tc_commit(smem_u32(&bars->drain2));
      mbar_wait_drain(smem_u32(&bars->drain2), 0, budget);
    }
  } else if (warp == 3) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kHelperRegsControl));
    // ================= P' producer: the slice of each (pass, slice) group, once MMA1 has
    // finished with the previous group's
    if (lane == 0 && ra < rb) {
      tma_prefetch_desc(&tmap_p);
      int q = 0;
      bool ok = true;
      for (long long c0 = ra; ok && c0 < rb; c0 += kChunk)
        for (int ph = 0; ok && ph < 2; ++ph)
          for (int s = 0; s < C; ++s, ++q) {
            if (!mbar_wait(smem_u32(&bars->p_empty), (uint32_t)((q & 1) ^ 1), status, budget)) {
              ok = false;
              break;
            }
            const uint32_t pf = smem_u32(&bars->p_full);
            mbar_arrive_expect_tx(pf, L::kPBytes);
            for (int b = 0; b < D / 64; ++b)
              tma_load_2d(sbase + L::oP + b * L::kSlot, &tmap_p, b * 64, s * kProtoSlice, pf);
          }
      if (q > 0) mbar_wait_drain(smem_u32(&bars->p_full), (uint32_t)((q - 1) & 1), budget);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHelperRegsSoftmax));
    // ================= softmax warpgroups (tile parity) + segment epilogues (warpgroup 0)
    const int wg = (warp >> 2) - 1;
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    TileIter base, it;
    base.init(tile_start, offsets, R, ra, rb);
    int nbw = 0, i2 = 0, useg = 0;
    long long run_g0 = 0;
    bool ok = true;
    for (long long c0 = ra; ok && c0 < rb; c0 += kChunk) {
      const int K = (int)(rb - c0 < kChunk ? rb - c0 : kChunk);
      for (int ph = 0; ok && ph < 2; ++ph) {
        for (int s = 0; ok && s < C; ++s) {
          const int pbase = s * kProtoSlice;
          const bool partial_slice = pbase + kProtoSlice > k_valid;
          it = base;
          int prev_u = -1;
          for (int tl = 0; tl < K; ++tl, it.next()) {
            const int sb = tl & 1;
            if (ph == 1 && (tl == 0 || it.u != prev_u)) run_g0 = it.g;
            prev_u = it.u;
            if (sb == wg) {
              if (!mbar_wait_warp(smem_u32(&bars->s_full[sb]), (uint32_t)(nbw & 1), status, budget)) {
                ok = false;
                break;
              }
              ++nbw;
              tc_fence_after();
              float v[kProtoSlice];
              load_scores(tmem + lane_off + (sb ? kColS1 : kColS0), v);
              // the scores are in registers: the buffer goes back to MMA1 at once, so the
              // score MMA of this warpgroup's next tile overlaps the exponentials below
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&bars->s_empty[sb]));
              if (partial_slice) {
#pragma unroll
                for (int c = 0; c < kProtoSlice; ++c)
                  if (pbase + c >= k_valid) v[c] = -INFINITY;
              }
              const bool valid = r < it.nvalid();
              float* lp = lsm + tl * kTileTokens + r;
              if (ph == 0) {
                // l = m + log2 sum 2^(s - m): no shift (m = 0) unless a lane's sum leaves
                // [2^-100, 2^100], as in the clustered kernel; only the sum is kept
                float m = 0.f;
                float z = sum_exp2(v, 0.f);
                if (!__all_sync(0xffffffffu, z >= 0x1p-100f && z <= 0x1p100f)) {
                  m = row_max(v);
                  z = sum_exp2(v, m);
                }
                const float l = valid ? m + lg2_approx(z) : 0.f;
                if (s == 0) {
                  *lp = l;
                } else {  // lse2 <- log2(2^lse2 + 2^l)
                  const float o = *lp;
                  const float hi = fmaxf(o, l), lo = fminf(o, l);
                  *lp = hi + lg2_approx(1.f + ex2_approx(lo - hi));
                }
              } else {
                // A = 2^(s - lse2) <= 1 directly (lse2 >= every score); rows past the
                // user's last token get A = 0
                const float lse2 = *lp;
                if (s == 0 && valid && lse_out != nullptr)
                  lse_out[it.t0() + r] = lse2 * 0.69314718055994530942f;
                const float off = valid ? -lse2 : -INFINITY;
                const uint64_t off2 = f2_pack(off, off);
                uint32_t pa0[32], pa1[32];
#pragma unroll
                for (int p = 0; p < 32; ++p) {
                  float a, b;
                  f2_unpack(f2_add(f2_pack(v[2 * p], v[2 * p + 1]), off2), a, b);
                  pa0[p] = cvt_bf16x2(ex2_approx(a), ex2_approx(b));
                  f2_unpack(f2_add(f2_pack(v[64 + 2 * p], v[64 + 2 * p + 1]), off2), a, b);
                  pa1[p] = cvt_bf16x2(ex2_approx(a), ex2_approx(b));
                }
                // A(i2) may overwrite the buffer once MMA2(i2 - 1) has read it; MMA1(i2) was
                // issued after MMA2(i2 - 4) completed, so this barrier is at most one phase
                // behind the awaited one
                if (!mbar_wait_warp(smem_u32(&bars->a_empty[(i2 - 1) & 3]),
                                    (uint32_t)(((i2 - 1) >> 2) & 1), status, budget)) {
                  ok = false;
                  break;
                }
                store_a_block(smem + L::abox(0, 0) + r * 128, r, pa0);
                store_a_block(smem + L::abox(0, 1) + r * 128, r, pa1);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->a_full));
              }
            }
            if (ph == 1) {
              if (wg == 0 && (tl == K - 1 || it.last())) {
                // ---- epilogue of the run that ends at this tile: U_s, mass_s into segment
                // (range G + b, user); stored by the segment's first run, added after that
                if (!mbar_wait_warp(smem_u32(&bars->u_full), (uint32_t)(useg & 1), status, budget)) {
                  ok = false;
                  break;
                }
                ++useg;
                tc_fence_after();
                const long long sgid = (long long)G + blockIdx.x + it.u;
                const bool seg_first = run_g0 == ra || run_g0 == tile_start[it.u];
                float* dst = part_u + ((size_t)sgid * k_pad + pbase + r) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                  uint32_t u32[32];
                  tmem_ld32_raw(tmem + lane_off + kColU + c * 32, u32);
                  tmem_wait_tie(u32);
#pragma unroll
                  for (int x = 0; x < 32; x += 4) {
                    float4 o = make_float4(__uint_as_float(u32[x]), __uint_as_float(u32[x + 1]),
                                           __uint_as_float(u32[x + 2]), __uint_as_float(u32[x + 3]));
                    float4* p4 = reinterpret_cast<float4*>(dst + c * 32 + x);
                    if (!seg_first) {
                      const float4 w4 = *p4;
                      o.x += w4.x; o.y += w4.y; o.z += w4.z; o.w += w4.w;
                    }
                    *p4 = o;
                  }
                }
                const float ms = tmem_ld1(tmem + lane_off + kColU + D);
                tc_wait_ld();
                float* pm = part_m + (size_t)sgid * k_pad + pbase + r;
                *pm = seg_first ? ms : *pm + ms;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->u_empty));
              }
              ++i2;
            }
          }
        }
      }
      base = it;
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // complete only after the clustered grid: work queued behind this grid sees its results
  griddep_wait();
}

template <int D, int NS, int NA>
cudaError_t launch_fwd_sm100_t(const FwdSm100Args& a, cudaStream_t stream) {
  auto kern = sa_fwd_sm100_kernel<D, NS, NA>;
  const size_t smem = FwdSmem<D, NS, NA>::bytes(a.C);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (a.C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.G * a.C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, *a.tmap_x, *a.tmap_p, a.offsets, a.R, a.k_valid, a.C,
                            a.k_pad, a.hdr, a.tile_start, a.part_u, a.part_m, a.lse, a.H,
                            a.share, a.budget);
}

template <int D, int NS, int NA>
cudaError_t max_clusters_t(int C, int* n) {
  auto kern = sa_fwd_sm100_kernel<D, NS, NA>;
  const size_t smem = FwdSmem<D, NS, NA>::bytes(C);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
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
  return cudaOccupancyMaxActiveClusters(n, kern, &cfg);
}

// X stages: 4 at d = 128 while the exchange slots leave room (C <= 8), else 3; 4 at d = 64.
int stages_for(int d, int C) { return d == 64 ? 4 : (C <= 8 ? 4 : 3); }

}  // namespace

cudaError_t fwd_sm100_max_clusters(int d, int C, int* n) {
  if (d == 64) return max_clusters_t<64, 4, 2>(C, n);
  return stages_for(d, C) == 4 ? max_clusters_t<128, 4, 1>(C, n) : max_clusters_t<128, 3, 1>(C, n);
}

// The helpers' share of the tiles balances the two grids: a cluster takes a tile in the
// time one helper takes kHelperCost of a slice of it (2 C passes of scores, C of them
// with the accumulate). Measured on a B200 at k = 1024, d = 128: alone, a helper tile
// takes 17.2 us against 1.27 us per tile for a cluster (1.70 per slice); beside the
// clusters (shared L2 and power) the fastest split was 1.86, 114/1024 of the tiles
// (shares 107 to 156 timed). A larger share makes the helpers finish last, a smaller one
// the clusters.
constexpr double kHelperCost = 1.86;

void fwd_sm100_helpers(int d, int C, int G, int sms, int* H, int* share) {
  *H = 0;
  *share = 0;
  const int free_sms = sms - G * C;
  if (d != 128 || C < 2 || free_sms < 4) return;
  const double rate = (double)free_sms / (C * kHelperCost);  // helper tiles per cluster tile
  *H = free_sms;
  *share = (int)std::lround(1024.0 * rate / (G + rate));
}

cudaError_t launch_fwd_sm100(const FwdSm100Args& a, cudaStream_t stream) {
  if (a.d == 64) return launch_fwd_sm100_t<64, 4, 2>(a, stream);
  cudaError_t e = stages_for(a.d, a.C) == 4 ? launch_fwd_sm100_t<128, 4, 1>(a, stream)
                                            : launch_fwd_sm100_t<128, 3, 1>(a, stream);
  if (e != cudaSuccess || a.H <= 0) return e;
  // the helper grid, queued behind the clustered one with programmatic serialization: it
  // starts once every cluster is resident (their CTAs trigger it after setup), so it can
  // only take the SMs that no cluster fits on, and it completes after the clustered grid
  auto kern = sa_fwd_sm100_helper_kernel<128>;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < kHelperRegsLaunch) return cudaErrorInvalidConfiguration;  // see the split
  const size_t smem = helper_smem_bytes<128>();
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.H);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, *a.tmap_x, *a.tmap_p, a.offsets, a.R, a.k_valid, a.C,
                            a.k_pad, a.hdr, a.tile_start, a.part_u, a.part_m, a.lse, a.G, a.H,
                            a.share, a.budget);
}

}  // namespace sa
