// Tensor-core GEMM building block (sm_100a): the finalize's W_v product, the backward's
// Gh, dW_v and log-sum-exp GEMMs, and the cross attention's projections and weight
// gradients.
//
//   C[128 x 128 tile] = sum over phases p, K tiles k of  A_p[m, k] . B_p[n, k]
//
// bf16 operands arrive by TMA in 128-byte-swizzled boxes; tcgen05.mma (kind::f16, fp32
// accumulate) runs from one thread into TMEM; four epilogue warps read the accumulator
// (thread = output row = TMEM lane) and apply one of the fused epilogues below. Each
// operand is either K-major (stored [M or N rows][K], K contiguous) or MN-major (stored
// [K rows][M or N], M/N contiguous), so A B^T, A^T B and A B are all one kernel.
//
// Row tiles are 128 consecutive rows of M.
//
// Epilogues:
//   kEpiStoreF32  out[row][n] = acc in fp32, or a split-K partial at split * split_stride
//   kEpiLse       dpart[row][2 tile + h] = log2 sum of 2^acc over half h of the tile
//                 (columns n < k_valid)
//   kEpiStoreBf16 out_bf16[row][n] = bf16(acc)
// Waits on mbarriers are bounded like every other kernel of the library.
#include <cuda.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStageBytes = (kBM + kBN) * kBK * 2;  // 32 KB
// pipeline stages: 3, or 2 when a CTA has at most 2 K tiles (then 3 CTAs fit per SM)
constexpr int kGemmThreads = 320;                   // producer, MMA, 8 epilogue warps

struct GemmParams {
  CUtensorMap ta[2], tb[2];
  int a_mn[2], b_mn[2];
  int k_tiles[2];
  int phases;
  int M, N;
  int splits;
  const WsHeader* hdr;
  float* out_f32;
  long long ld_out;
  long long split_stride;
  __nv_bfloat16* out_bf16;
  int k_valid;
  float* dpart;
  int dpart_ld;
  long long budget;
};

template <int NST>
struct GemmBars {
  uint64_t full[NST], empty[NST], done, drain;
  uint32_t tmem_base;
};

// One operand tile (128 rows of M or N by 64 of K) of the given layout into smem.
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* tm, int mn_major,
                                             int mn0, int k0, uint32_t bar) {
  if (!mn_major) {
    tma_load_2d(dst, tm, k0, mn0, bar);  // box {64 K, 128 rows}
  } else {
    tma_load_2d(dst, tm, mn0, k0, bar);              // box {64 M/N, 64 K}
    tma_load_2d(dst + 8192, tm, mn0 + 64, k0, bar);  // the second 64 M/N columns
  }
}

// Shared-memory descriptor of K step ks (16 wide) of an operand tile.
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int mn_major, int ks) {
  return mn_major ? smem_desc(base + ks * 2048, 8192, 1024, kSwizzle128B)
                  : smem_desc(base + ks * 32, 16, 1024, kSwizzle128B);
}

template <int EPI, int NST>
__global__ void __launch_bounds__(kGemmThreads, (NST == 2 && EPI != kEpiStoreF32) ? 3 : 2)
sa_gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr int kStages = NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  GemmBars<NST>* bars = reinterpret_cast<GemmBars<NST>*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = const_cast<int*>(&p.hdr->status);

  // ---- which output tile: blockIdx.x = m_tile * n_tiles + n_tile, so the n_tiles CTAs
  // that share one block of A rows run together and read it from DRAM once (L2 after)
  const unsigned n_tiles = (unsigned)(p.N + kBN - 1) / kBN;
  const int n_tile = (int)(blockIdx.x % n_tiles);
  const long long m_tile = (long long)(blockIdx.x / n_tiles);
  const int row0 = (int)(m_tile * kBM);
  const int nrows = min(kBM, p.M - row0);
  if (nrows <= 0) return;
  const int n0 = n_tile * kBN;
  // K tiles of this CTA: phase 0 is split evenly across gridDim.y; phase 1 is not split
  const int z = blockIdx.y;
  const int kt0 = (int)((long long)p.k_tiles[0] * z / p.splits);
  const int kt1 = (int)((long long)p.k_tiles[0] * (z + 1) / p.splits);
  const int total_kt = (kt1 - kt0) + (p.phases > 1 ? p.k_tiles[1] : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->done), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ================= TMA producer
    if (lane == 0 && total_kt > 0) {
      for (int ph = 0; ph < p.phases; ++ph) {
        tma_prefetch_desc(&p.ta[ph]);
        tma_prefetch_desc(&p.tb[ph]);
      }
      for (int j = 0; j < total_kt; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(smem_u32(&bars->empty[st]), (uint32_t)(((j / kStages) & 1) ^ 1), status,
                       p.budget))
          break;
        const int ph = j < kt1 - kt0 ? 0 : 1;
        const int kt = ph == 0 ? kt0 + j : j - (kt1 - kt0);
        const uint32_t fb = smem_u32(&bars->full[st]);
        mbar_arrive_expect_tx(fb, kStageBytes);
        const uint32_t sa = sbase + st * kStageBytes;
        load_operand(sa, &p.ta[ph], p.a_mn[ph], row0, kt * kBK, fb);
        load_operand(sa + kBM * kBK * 2, &p.tb[ph], p.b_mn[ph], n0, kt * kBK, fb);
      }
      // the last stages' loads must land before exit
      for (int j = total_kt > kStages ? total_kt - kStages : 0; j < total_kt; ++j)
        mbar_wait_drain(smem_u32(&bars->full[j % kStages]), (uint32_t)((j / kStages) & 1), p.budget);
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0 && total_kt > 0) {
      const uint32_t idesc0 = idesc_bf16_f32(kBM, kBN, p.a_mn[0], p.b_mn[0]);
      const uint32_t idesc1 = idesc_bf16_f32(kBM, kBN, p.a_mn[1], p.b_mn[1]);
      bool ok = true;
      for (int j = 0; j < total_kt && ok; ++j) {
        const int st = j % kStages;
        ok = mbar_wait(smem_u32(&bars->full[st]), (uint32_t)((j / kStages) & 1), status, p.budget);
        if (!ok) break;
        tc_fence_after();
        const int ph = j < kt1 - kt0 ? 0 : 1;
        const uint32_t sa = sbase + st * kStageBytes, sb = sa + kBM * kBK * 2;
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks)
          tc_mma_f16(tmem, operand_desc(sa, p.a_mn[ph], ks), operand_desc(sb, p.b_mn[ph], ks),
                     ph ? idesc1 : idesc0, (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(smem_u32(&bars->empty[st]));
      }
      tc_commit(smem_u32(&bars->done));
      mbar_wait_drain(smem_u32(&bars->done), 0, p.budget);
    }
  } else {
    // ================= epilogue: thread = output row (TMEM lane), in 32-column chunks.
    // Global traffic goes through a per-warp staging block in the (now idle) pipeline
    // shared memory, so every load and store below is a full, coalesced row segment.
    // Two warps per TMEM lane quadrant: epilogue warp e (0..7) takes rows of quadrant
    // e & 3 and the column half e >> 2 of the tile.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float* stg = reinterpret_cast<float*>(smem) + (warp - 2) * (32 * 33);  // [32][33]
    const bool have = total_kt > 0 &&
                      mbar_wait_warp(smem_u32(&bars->done), 0, status, p.budget);
    if (have) {
      tc_fence_after();
      const bool valid = r < nrows;
      const long long row = (long long)row0 + r;
      const int wrow0 = q * 32;  // first tile row of this warp
      float lmax = -INFINITY, lsum = 0.f;
#pragma unroll 1
      for (int c = half * 2; c < half * 2 + 2; ++c) {
        uint32_t u[32];
        tmem_ld32_raw(tmem + lane_off + c * 32, u);
        tmem_wait_tie(u);
        const int nb = n0 + c * 32;
        if (nb >= p.N) continue;  // warp-uniform
        float v[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = __uint_as_float(u[x]);
        if (EPI == kEpiLse) {
          float cm = -INFINITY;
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (nb + x < p.k_valid) cm = fmaxf(cm, v[x]);
          if (cm > -INFINITY) {
            float cs = 0.f;
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (nb + x < p.k_valid) cs += ex2_approx(v[x] - cm);
            const float nm = fmaxf(lmax, cm);
            lsum = lsum * ex2_approx(lmax - nm) + cs * ex2_approx(cm - nm);
            lmax = nm;
          }
          continue;
        }
        // stage this warp's 32 x 32 outputs, then store them row by row
        __syncwarp();
#pragma unroll
        for (int x = 0; x < 32; ++x) stg[lane * 33 + x] = v[x];
        __syncwarp();
        if (EPI == kEpiStoreF32) {
          float* dst = p.out_f32 + (long long)z * p.split_stride;
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + (lane >> 3), cc = (lane & 7) * 4;
            if (wrow0 + rr < nrows && nb + cc < p.N)
              *reinterpret_cast<float4*>(dst + (row0 + wrow0 + rr) * p.ld_out + nb + cc) =
                  make_float4(stg[rr * 33 + cc], stg[rr * 33 + cc + 1], stg[rr * 33 + cc + 2],
                              stg[rr * 33 + cc + 3]);
          }
        } else {  // bf16 output
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int rr = it * 8 + (lane >> 2), cc = (lane & 3) * 8;
            if (wrow0 + rr < nrows && nb + cc < p.N) {
              const float* sr = stg + rr * 33 + cc;
              *reinterpret_cast<uint4*>(p.out_bf16 + (row0 + wrow0 + rr) * p.ld_out + nb + cc) =
                  make_uint4(cvt_bf16x2(sr[0], sr[1]), cvt_bf16x2(sr[2], sr[3]),
                             cvt_bf16x2(sr[4], sr[5]), cvt_bf16x2(sr[6], sr[7]));
            }
          }
        }
      }
      if (EPI == kEpiLse && valid)
        p.dpart[row * p.dpart_ld + 2 * n_tile + half] =
            lmax > -INFINITY ? lmax + lg2_approx(lsum) : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBN);
  }
}

// Row-major bf16 matrix [rows][cols] with boxes of box_cols x box_rows (128B swizzle).
bool make_operand_map(CUtensorMap* m, const GemmOperandDesc& o) {
  auto fn = tmap_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {o.cols, o.rows};
  const cuuint64_t strides[1] = {o.cols * 2};
  const cuuint32_t box[2] = {64, o.mn_major ? 64u : 128u};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(o.base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int NST>
cudaError_t launch_st(const GemmParams& p, dim3 grid, cudaStream_t s) {
  static_assert(8 * (32 * 33) * 4 <= NST * kStageBytes, "epilogue staging fits the stages");
  const size_t smem = 1024 + NST * kStageBytes + sizeof(GemmBars<NST>);
  cudaError_t e = cudaFuncSetAttribute(sa_gemm_kernel<EPI, NST>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  sa_gemm_kernel<EPI, NST><<<grid, kGemmThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_t(const GemmParams& p, dim3 grid, cudaStream_t s) {
  const int kt_max = (p.k_tiles[0] + p.splits - 1) / p.splits + (p.phases > 1 ? p.k_tiles[1] : 0);
  return kt_max <= 2 ? launch_st<EPI, 2>(p, grid, s) : launch_st<EPI, 3>(p, grid, s);
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
  GemmParams p = {};
  for (int ph = 0; ph < g.phases; ++ph) {
    if (!make_operand_map(&p.ta[ph], g.a[ph]) || !make_operand_map(&p.tb[ph], g.b[ph]))
      return cudaErrorInvalidValue;
    p.a_mn[ph] = g.a[ph].mn_major ? 1 : 0;
    p.b_mn[ph] = g.b[ph].mn_major ? 1 : 0;
    p.k_tiles[ph] = g.k_tiles[ph];
  }
  if (g.phases == 1) {
    p.ta[1] = p.ta[0];
    p.tb[1] = p.tb[0];
  }
  p.phases = g.phases;
  p.M = g.M;
  p.N = g.N;
  p.splits = g.splits < 1 ? 1 : g.splits;
  p.hdr = g.hdr;
  p.out_f32 = g.out_f32;
  p.ld_out = g.ld_out;
  p.split_stride = g.split_stride;
  p.out_bf16 = g.out_bf16;
  p.k_valid = g.k_valid;
  p.dpart = g.dpart;
  p.dpart_ld = g.dpart_ld;
  p.budget = kDefaultWaitBudget;
  const long long tiles = (long long)g.m_tiles_bound * ((g.N + kBN - 1) / kBN);
  if (tiles > 0x7FFFFFFFLL || p.splits > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)tiles, (unsigned)p.splits);
  if (grid.x == 0) return cudaSuccess;
  switch (g.epi) {
    case kEpiStoreF32: return launch_t<kEpiStoreF32>(p, grid, s);
    case kEpiLse: return launch_t<kEpiLse>(p, grid, s);
    case kEpiStoreBf16: return launch_t<kEpiStoreBf16>(p, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
