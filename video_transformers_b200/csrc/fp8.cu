// fp8.cu -- e4m3 query and key operands for the FP8 attention path (news
// review "[Paper] PSA ...", Practical Implications: mixed FP16 / FP8
// precision; the pages give no scheme).  Each query row is scaled by
// 448 / max|q_row|; every key of a KV head, at every pyramid level, by
// 448 / max|K| over the head's level 0 (a mean never exceeds the largest
// magnitude it averages, so no level saturates).  Scales and the scaled
// values are fp32; each is rounded to the nearest e4m3 value, ties to even,
// saturating at +-448 (cvt.rn.satfinite).
//
// The values of the FP8 probability path are coded like the keys, with
// their own per-head scale.
//
// kabsmax_kernel   one CTA per KV head: max |K| over level 0.
// quant_rows_kernel  one warp per query row: its max, scale and codes.
// quant_head_kernel  every key of every level, with its head's multiplier.
// head_scale_kernel  max / 448 per head (after the codes are written).
#include <cuda_bf16.h>

#include "internal.h"

namespace psa {
namespace {

constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(1024) kabsmax_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ am,
                                                       int64_t per_head) {
  __shared__ float wmax[32];
  const int64_t bh = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(k + bh * per_head);
  const int64_t n16 = per_head / 8;
  float m = 0.f;
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < blockDim.x / 32 ? wmax[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) am[bh] = m;
  }
}

// one warp per row of d channels (d = 64 or 128): 2 or 4 per lane
template <int D>
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ codes,
                                                         float* __restrict__ scale, int64_t rows) {
  constexpr int PER = D / 32;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float v[PER];
  if (PER == 4) {
    const uint2 u = reinterpret_cast<const uint2*>(x + row * D)[lane];
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x; v[1] = a.y; v[PER > 2 ? 2 : 0] = b.x; v[PER > 3 ? 3 : 0] = b.y;
  } else {
    const uint32_t u = reinterpret_cast<const uint32_t*>(x + row * D)[lane];
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
    v[0] = a.x; v[PER > 1 ? 1 : 0] = a.y;
  }
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float inv = m > 0.f ? kE4m3Max / m : 0.f;
  if (PER == 4) {
    const uint32_t c = static_cast<uint32_t>(e4m3x2(v[0] * inv, v[1] * inv)) |
                       (static_cast<uint32_t>(e4m3x2(v[PER > 2 ? 2 : 0] * inv, v[PER > 3 ? 3 : 0] * inv)) << 16);
    reinterpret_cast<uint32_t*>(codes + row * D)[lane] = c;
  } else {
    reinterpret_cast<uint16_t*>(codes + row * D)[lane] = e4m3x2(v[0] * inv, v[PER > 1 ? 1 : 0] * inv);
  }
  if (lane == 0) scale[row] = m / kE4m3Max;
}

// every element of one level ([BH][n][d], bf16) with its head's multiplier
__global__ void __launch_bounds__(256) quant_head_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ codes,
                                                         const float* __restrict__ am, int64_t per_head, int64_t total) {
  const int64_t n8 = total / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t bh = (i * 8) / per_head;
    const float m = am[bh];
    const float inv = m > 0.f ? kE4m3Max / m : 0.f;
    const uint4 u = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t out[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * j]));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * j + 1]));
      out[j] = static_cast<uint32_t>(e4m3x2(a.x * inv, a.y * inv)) |
               (static_cast<uint32_t>(e4m3x2(b.x * inv, b.y * inv)) << 16);
    }
    reinterpret_cast<uint2*>(codes)[i] = make_uint2(out[0], out[1]);
  }
}

__global__ void head_scale_kernel(float* am, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) am[i] = am[i] / kE4m3Max;
}

int grid_cap(int64_t work, int threads) {
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_quantize_heads_fp8(const void* x, const void* x_pyr, const size_t* level_off, int64_t BH, int N,
                                     int d, int levels, uint8_t* x8, uint8_t* x8_pyr, float* scale, cudaStream_t s) {
  // scale holds the per-head maxima until every level is coded
  kabsmax_kernel<<<static_cast<unsigned>(BH), 1024, 0, s>>>(static_cast<const __nv_bfloat16*>(x), scale,
                                                            static_cast<int64_t>(N) * d);
  const int64_t t0 = BH * N * d;
  quant_head_kernel<<<grid_cap(t0 / 8, 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), x8, scale,
                                                          static_cast<int64_t>(N) * d, t0);
  for (int l = 1; l < levels; ++l) {
    const int64_t per = static_cast<int64_t>(N >> l) * d;
    const int64_t tl = BH * per;
    quant_head_kernel<<<grid_cap(tl / 8, 256), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(static_cast<const char*>(x_pyr) + level_off[l] * 2), x8_pyr + level_off[l],
        scale, per, tl);
  }
  head_scale_kernel<<<static_cast<unsigned>((BH + 255) / 256), 256, 0, s>>>(scale, static_cast<int>(BH));
  return cudaGetLastError();
}

cudaError_t launch_quantize_qk_fp8(const void* q, const void* k, const void* k_pyr, const size_t* level_off,
                                   int64_t BHq, int64_t BHkv, int N, int d, int levels, uint8_t* q8, float* q_scale,
                                   uint8_t* k8, uint8_t* k8_pyr, float* k_scale, cudaStream_t s) {
  const int64_t qrows = BHq * N;
  const int64_t warps_per_cta = 8;
  const unsigned qgrid = static_cast<unsigned>((qrows + warps_per_cta - 1) / warps_per_cta);
  if (d == 128)
    quant_rows_kernel<128><<<qgrid, 32 * warps_per_cta, 0, s>>>(static_cast<const __nv_bfloat16*>(q), q8, q_scale, qrows);
  else
    quant_rows_kernel<64><<<qgrid, 32 * warps_per_cta, 0, s>>>(static_cast<const __nv_bfloat16*>(q), q8, q_scale, qrows);
  return launch_quantize_heads_fp8(k, k_pyr, level_off, BHkv, N, d, levels, k8, k8_pyr, k_scale, s);
}

}  // namespace psa
