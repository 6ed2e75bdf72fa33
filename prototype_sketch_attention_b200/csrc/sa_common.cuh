// Device-side helpers shared by the Sketch Attention kernels (sm_100a).
//
// Thin inline-PTX wrappers for mbarriers, TMA, tcgen05 (TMEM allocation, MMA,
// commit, loads) and cluster distributed shared memory. Every wait on an mbarrier
// is bounded: after `budget` SM clocks it latches SA_ERR_TIMEOUT in the workspace
// status word and returns false, and callers leave their loops. No kernel spins
// forever, and none traps.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "sa_sketch.h"

namespace sa {

// ---------------------------------------------------------------- workspace header
// The first 256 bytes of every workspace: the device status word and scalars that
// the schedule kernel computes for later kernels.
struct WsHeader {
  int status;          // SA_OK, or the first device-side error latched this call
  int pad0;
  long long total_tiles;  // sum over users of ceil(n_u / 128)
  long long pad[30];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int kTileTokens = 128;  // tokens per tile (tcgen05 M and the split unit)
constexpr long long kDefaultWaitBudget = 4000000000LL;  // SM clocks (about 2 s)

__device__ __forceinline__ void latch_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ int read_status(const int* status) {
  return *reinterpret_cast<const volatile int*>(status);
}

// ---------------------------------------------------------------- shared memory / mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}"
               ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}"
               ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Acquire at cluster scope: used for barriers that peers complete (st.async).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity. Returns false (after latching
// SA_ERR_TIMEOUT unless another error is already latched) if the budget runs out
// or if another thread has already latched an error.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* status,
                                          long long budget) {
  if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  uint32_t iter = 0;
  while (true) {
    if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((++iter & 63u) == 0u) {
      if (read_status(status) != 0) return false;
      if (clock64() - t0 > budget) {
        latch_status(status, SA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform variant for code that continues with .sync.aligned instructions:
// every lane of the warp gets the same answer.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, int* status,
                                               long long budget) {
  return __all_sync(0xffffffffu, mbar_wait<kCluster>(bar, parity, status, budget));
}

// Same, but ignores errors latched by others: used on the way out to drain copies
// this thread issued itself.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, long long budget) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- cluster
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// 16-byte remote store into a peer's shared memory that completes `bytes` (16) of
// the transaction count of the peer's mbarrier at `rbar`.
__device__ __forceinline__ void st_async_v4(uint32_t raddr, float a, float b, float c, float d,
                                            uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(raddr), "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(__float_as_uint(c)),
        "r"(__float_as_uint(d)), "r"(rbar)
      : "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled load of one box into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(dst_smem), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on an mbarrier of this CTA when all previously issued tcgen05 ops of
// this thread have completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 columns into raw registers (no wait); pair with tmem_wait_tie.
__device__ __forceinline__ void tmem_ld32_raw(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// tcgen05.wait::ld that also carries the loaded registers as in/out operands, so no
// use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_tie(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// 32 lanes x 16 columns into raw registers (no wait); pair with tmem_wait16.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// tcgen05.wait::ld tied to 16 loaded registers (see tmem_wait_tie).
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15])
      :
      : "memory");
}

// 32 lanes x 16 columns from registers (complete with tcgen05.wait::st).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
        "r"(r[14]), "r"(r[15])
      : "memory");
}

// Empty asm that carries 32 registers through: a use after it cannot be scheduled before
// it (pairs with tmem_wait_tie when two tcgen05.ld share one wait).
__device__ __forceinline__ void tie32(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]));
}

// Shared-memory matrix descriptor for tcgen05 (start, leading and stride byte
// offsets in 16-byte units; version 1; swizzle mode in bits 61..63).
enum : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2, kSwizzle32B = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version for sm_100
  d |= (uint64_t)(swizzle & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
// a_mn / b_mn: 1 if that operand is MN-major (0 = K-major).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16)
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// ---------------------------------------------------------------- packed fp32 (sm_100)
// Two fp32 lanes in one 64-bit register pair: one instruction, two results.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Pull one TMA box into L2 ahead of its load (no shared memory involved).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];"
               ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y) : "memory");
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- tile ranges
// The forward splits the token tiles [0, T) into G cluster ranges over [0, T1) and H helper
// ranges over [T1, T) (helper CTAs run on the SMs that no cluster fits on). The helpers'
// share is `share` / 1024 of the tiles: Th = floor(T share / 1024), T1 = T - Th, except
// that the helpers take no tiles (Th = 0) unless each gets at least kHelperMinTiles: a
// helper pays a fixed cost per (pass, slice) group of a chunk, which only full chunks
// amortise. Range g < G is [g T1 / G, (g + 1) T1 / G); range G + b is
// [T1 + b Th / H, T1 + (b + 1) Th / H). The forward kernels and the finalize take the
// ranges from this one definition.
constexpr long long kHelperMinTiles = 32;
__device__ __forceinline__ long long helper_tiles(long long T, int H, int share) {
  const long long th = H > 0 ? (T * share) >> 10 : 0;
  return th >= kHelperMinTiles * H ? th : 0;
}
struct TileRanges {
  long long T1, Th;
  int G, H;
  __device__ TileRanges(long long T, int G_, int H_, int share)
      : T1(T - helper_tiles(T, H_, share)), Th(helper_tiles(T, H_, share)), G(G_), H(H_) {}
  __device__ long long start(long long g) const {
    return g <= G ? g * T1 / G : T1 + (g - G) * Th / H;
  }
  // the range holding tile x (0 <= x < T1 + Th); empty ranges are never returned
  __device__ int of_tile(long long x) const {
    const bool helper = x >= T1;
    const long long base = helper ? T1 : 0, n = helper ? Th : T1;
    const int m = helper ? H : G;
    const long long y = x - base;
    long long g = y * m / n;
    if (g >= m) g = m - 1;
    while (g + 1 < m && (g + 1) * n / m <= y) ++g;
    while (g > 0 && g * n / m > y) --g;
    return (int)g + (helper ? G : 0);
  }
};

// Programmatic dependent launch. launch_dependents: the grid queued after this one with
// the programmatic stream serialization attribute may start once every CTA of this grid
// has executed it (or exited). wait: blocks until the grids this one depends on that way
// have completed and their memory operations are visible.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Token tile -> user lookup: the user whose tile range contains tile `g`
// (tile_start is the exclusive prefix sum of per-user tile counts, length R+1).
__device__ __forceinline__ int user_of_tile(const long long* tile_start, int R, long long g) {
  int lo = 0, hi = R;  // invariant: tile_start[lo] <= g < tile_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

// Walks the tiles [a, b) of the global tile sequence (users' tiles concatenated).
// Tile indices fit in 32 bits: n_total < 2^31 tokens gives fewer than 2^31 tiles.
struct TileIter {
  // Walks the tiles [g0, end) of the concatenated per-user tile lists. The current
  // user's tile and token bounds live in registers; global memory (tile_start,
  // offsets) is read only when the walk crosses into the next user, so the per-tile
  // queries below cost no memory round trip.
  const long long* ts;
  const int64_t* off;
  int g, end, u;
  int ts_u1;    // first tile of the next user (tiles of user u end there)
  int t0b;      // first token of tile g is t0b + 128 g (n_total < 2^31)
  int tok_end;  // one past the last token of user u
  __device__ void init(const long long* ts_, const int64_t* off_, int R, long long a_,
                       long long b_) {
    ts = ts_; off = off_; g = (int)a_; end = (int)b_; u = 0;
    ts_u1 = t0b = tok_end = 0;
    if (a_ < b_) {
      u = user_of_tile(ts, R, a_);
      const int ts_u = (int)ts[u];
      ts_u1 = (int)ts[u + 1];
      t0b = (int)off[u] - ts_u * kTileTokens;
      tok_end = (int)off[u + 1];
    }
  }
  __device__ bool valid() const { return g < end; }
  __device__ long long t0() const { return (long long)t0b + g * kTileTokens; }
  __device__ int nvalid() const {
    const int n = tok_end - (t0b + g * kTileTokens);
    return n >= kTileTokens ? kTileTokens : n;
  }
  __device__ bool last() const { return g == end - 1 || g == ts_u1 - 1; }
  __device__ void next() {
    ++g;
    if (g < end) {
      while (ts_u1 <= g) {  // next user (users without tiles are skipped)
        ++u;
        t0b = tok_end - ts_u1 * kTileTokens;
        ts_u1 = (int)ts[u + 1];
        tok_end = (int)off[u + 1];
      }
    }
  }
};

}  // namespace sa
