// Sketch cache codec: fp32 sketches packed for the cache between requests, and back.
//
// The sketch is user-only and is reused across candidates and requests ("100,000
// videos in your pocket" blog, section "3. The system makes it cheap enough to
// matter", low-rank caching); the pages name no storage format. Two formats:
//   bf16: each value rounded to the nearest bfloat16 (ties to even).
//   fp8:  per row a scale s = max |row| / 448 (1 for an all-zero row), computed in fp32;
//         each value x / s (fp32 IEEE division) rounded to the nearest FP8 E4M3 value,
//         saturating at 448 (finite-only variant); zeros stored as +0. Decode: code * s.
// Both are bound by HBM traffic (5 bytes per value for fp8 packing, 6 for bf16), so the
// kernels are grid-stride loops with 16-byte loads, one row per warp (d / 4 lanes) for
// fp8, whose scale needs the row's maximum.
#include <cuda_fp8.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {
namespace {

constexpr float kE4m3Max = 448.0f;

__global__ void pack_bf16_kernel(const float4* __restrict__ x, long long n4,
                                 uint2* __restrict__ out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 v = x[i];
    out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

__global__ void unpack_bf16_kernel(const uint2* __restrict__ in, long long n4,
                                   float4* __restrict__ out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const uint2 b = in[i];
    out[i] = make_float4(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u),
                         __uint_as_float(b.y << 16), __uint_as_float(b.y & 0xFFFF0000u));
  }
}

__device__ __forceinline__ uint32_t e4m3(float y) {
  uint32_t c = __nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
  return (c & 0x7Fu) == 0 ? 0u : c;  // +0 for zero (the sign of a zero is not kept)
}

// One row per LANES lanes (LANES = d / 4), 4 values per lane.
template <int LANES>
__global__ void pack_fp8_kernel(const float4* __restrict__ x, long long rows,
                                uint32_t* __restrict__ codes, float* __restrict__ scales) {
  const int lane = threadIdx.x & (LANES - 1);
  const long long g0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / LANES;
  const long long gs = (gridDim.x * (long long)blockDim.x) / LANES;
  const unsigned mask = LANES == 32 ? 0xffffffffu
                                    : (0xffffu << (threadIdx.x & 16));  // this half-warp
  for (long long r = g0; r < rows; r += gs) {
    const float4 v = x[r * LANES + lane];
    float m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = LANES / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(mask, m, o, LANES));
    const float s = m > 0.f ? __fdiv_rn(m, kE4m3Max) : 1.0f;
    codes[r * LANES + lane] = e4m3(__fdiv_rn(v.x, s)) | (e4m3(__fdiv_rn(v.y, s)) << 8) |
                              (e4m3(__fdiv_rn(v.z, s)) << 16) | (e4m3(__fdiv_rn(v.w, s)) << 24);
    if (lane == 0) scales[r] = s;
  }
}

__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t ef = (b >> 3) & 0xFu, mant = b & 0x7u;
  // exact: ef = 0 holds the subnormals mant * 2^-9, else (8 + mant) * 2^(ef - 10)
  const float mag = ef == 0 ? (float)mant * 0x1p-9f
                            : (float)(8u + mant) * __uint_as_float((ef - 10u + 127u) << 23);
  return (b & 0x80u) ? -mag : mag;
}

template <int LANES>
__global__ void unpack_fp8_kernel(const uint32_t* __restrict__ codes,
                                  const float* __restrict__ scales, long long rows,
                                  float4* __restrict__ out) {
  const int lane = threadIdx.x & (LANES - 1);
  const long long g0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / LANES;
  const long long gs = (gridDim.x * (long long)blockDim.x) / LANES;
  for (long long r = g0; r < rows; r += gs) {
    const uint32_t c = codes[r * LANES + lane];
    const float s = scales[r];
    out[r * LANES + lane] = make_float4(e4m3_value(c & 0xFFu) * s, e4m3_value((c >> 8) & 0xFFu) * s,
                                        e4m3_value((c >> 16) & 0xFFu) * s, e4m3_value(c >> 24) * s);
  }
}

unsigned grid_for(long long work, int per_block) {
  long long b = (work + per_block - 1) / per_block;
  if (b > 148LL * 16) b = 148LL * 16;
  return (unsigned)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_sketch_pack(const float* S, long long rows, int d, int format, void* codes,
                               float* scales, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const long long n4 = rows * d / 4;
  if (format == 0) {
    pack_bf16_kernel<<<grid_for(n4, 256), 256, 0, s>>>(reinterpret_cast<const float4*>(S), n4,
                                                        static_cast<uint2*>(codes));
  } else if (d == 128) {
    pack_fp8_kernel<32><<<grid_for(rows, 8), 256, 0, s>>>(reinterpret_cast<const float4*>(S), rows,
                                                          static_cast<uint32_t*>(codes), scales);
  } else {
    pack_fp8_kernel<16><<<grid_for(rows, 16), 256, 0, s>>>(reinterpret_cast<const float4*>(S), rows,
                                                           static_cast<uint32_t*>(codes), scales);
  }
  return cudaGetLastError();
}

cudaError_t launch_sketch_unpack(const void* codes, const float* scales, long long rows, int d,
                                 int format, float* S, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const long long n4 = rows * d / 4;
  if (format == 0) {
    unpack_bf16_kernel<<<grid_for(n4, 256), 256, 0, s>>>(static_cast<const uint2*>(codes), n4,
                                                          reinterpret_cast<float4*>(S));
  } else if (d == 128) {
    unpack_fp8_kernel<32><<<grid_for(rows, 8), 256, 0, s>>>(static_cast<const uint32_t*>(codes),
                                                            scales, rows, reinterpret_cast<float4*>(S));
  } else {
    unpack_fp8_kernel<16><<<grid_for(rows, 16), 256, 0, s>>>(static_cast<const uint32_t*>(codes),
                                                             scales, rows, reinterpret_cast<float4*>(S));
  }
  return cudaGetLastError();
}

}  // namespace sa
