// pyramid.cu -- stage 1 of the PSA forward path: the KV pyramid
// ("psa-pyramid-sparse-attention" skill page, Core Technique: level l is the
// KV pooled by 2^l; summary article "PSA: Pyramid Sparse Attention ...",
// Method: the pyramid is built by repeated 1D mean pooling), plus the
// intra-block cosine statistic used by the pooling constraint (same
// article, Method and Results), plus the fp32 -> bf16 operand cast.
//
// Bandwidth kernel: one thread owns one 16-byte channel vector of a run of
// G = 2^(L-1) consecutive tokens, sums pairs in fp32 registers (a pairwise
// tree, so level l+1 is built from level l's unrounded sums) and rounds each
// level once to the storage type.  Reads K and V once, writes 1 - 2^-(L-1)
// of their size.
#include <cuda_bf16.h>

#include "internal.h"

namespace psa {
namespace {

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const void* p, float* x) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  __device__ static void store(void* p, const float* x) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = raw;
  }
};
template <>
struct Vec<float> {
  static constexpr int kN = 4;
  __device__ static void load(const void* p, float* x) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  }
  __device__ static void store(void* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

// G tokens per thread-run: 2 (L=2), 4 (L=3) or 8 (L=4).
template <typename T, int G>
__global__ void __launch_bounds__(256) pyramid_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                      char* __restrict__ kp, char* __restrict__ vp,
                                                      int64_t BH, int N, int d, size_t off1,
                                                      size_t off2, size_t off3) {
  constexpr int V = Vec<T>::kN;
  const int vecs = d / V;
  const int64_t runs = static_cast<int64_t>(N / G);
  const int64_t per_tensor = BH * runs * vecs;
  const int64_t total = 2 * per_tensor;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int tensor = u >= per_tensor;
    const int64_t rem = u - tensor * per_tensor;
    const int cv = static_cast<int>(rem % vecs);
    const int64_t run = rem / vecs;                 // bh * runs + r
    const int64_t bh = run / runs;
    const int64_t r = run - bh * runs;
    const T* src = (tensor ? v : k) + ((bh * N + r * G) * d + cv * V);
    char* dst = tensor ? vp : kp;

    float x[G][V];
#pragma unroll
    for (int t = 0; t < G; ++t) Vec<T>::load(src + static_cast<int64_t>(t) * d, x[t]);

    // level 1: pair sums
    float s1[G / 2][V];
#pragma unroll
    for (int t = 0; t < G / 2; ++t) {
      float y[V];
#pragma unroll
      for (int c = 0; c < V; ++c) {
        s1[t][c] = x[2 * t][c] + x[2 * t + 1][c];
        y[c] = s1[t][c] * 0.5f;
      }
      const int64_t row = bh * (N / 2) + r * (G / 2) + t;
      Vec<T>::store(dst + off1 + (row * d + cv * V) * sizeof(T), y);
    }
    if constexpr (G >= 4) {
      float s2[G / 4][V];
#pragma unroll
      for (int t = 0; t < G / 4; ++t) {
        float y[V];
#pragma unroll
        for (int c = 0; c < V; ++c) {
          s2[t][c] = s1[2 * t][c] + s1[2 * t + 1][c];
          y[c] = s2[t][c] * 0.25f;
        }
        const int64_t row = bh * (N / 4) + r * (G / 4) + t;
        Vec<T>::store(dst + off2 + (row * d + cv * V) * sizeof(T), y);
      }
      if constexpr (G >= 8) {
        float y[V];
#pragma unroll
        for (int c = 0; c < V; ++c) y[c] = (s2[0][c] + s2[1][c]) * 0.125f;
        const int64_t row = bh * (N / 8) + r;
        Vec<T>::store(dst + off3 + (row * d + cv * V) * sizeof(T), y);
      }
    }
  }
}

// One CTA (8 warps) per (bh, KV block).  Each warp normalises whole keys
// (lane c holds channels c*C .. c*C+C-1), the CTA sums the unit vectors and
// returns (|sum u|^2 - sum |u|^2) / (n (n - 1)), which equals the mean of
// cos(k_i, k_j) over ordered pairs i != j.
template <typename T, int D>
__global__ void __launch_bounds__(256) blockcos_kernel(const T* __restrict__ k, float* __restrict__ out,
                                                       int N, int block, int nkb) {
  constexpr int C = D / 32;
  __shared__ float part[8][D];
  __shared__ double red[8];
  __shared__ double sqs[8];
  const int J = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = J * block, t1 = min(t0 + block, N);
  const int n = t1 - t0;
  float acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  double sq = 0.0;
  for (int t = t0 + warp; t < t1; t += 8) {
    const T* p = k + (bh * N + t) * D + lane * C;
    float x[C];
#pragma unroll
    for (int c = 0; c < C; ++c) x[c] = static_cast<float>(p[c]);
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) ss = fmaf(x[c], x[c], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = fmaf(x[c], inv, acc[c]);
    sq += static_cast<double>(ss) * inv * inv;
  }
#pragma unroll
  for (int c = 0; c < C; ++c) part[warp][lane * C + c] = acc[c];
  if (lane == 0) sqs[warp] = sq;
  __syncthreads();
  double v2 = 0.0;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += part[w][c];
    v2 += s * s;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v2 += __shfl_xor_sync(0xffffffffu, v2, o);
  if (lane == 0) red[warp] = v2;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0, sqt = 0.0;
    for (int w = 0; w < 8; ++w) { tot += red[w]; sqt += sqs[w]; }
    out[bh * nkb + J] = n == 1 ? 1.0f : static_cast<float>((tot - sqt) / (static_cast<double>(n) * (n - 1)));
  }
}

__global__ void cast_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, int64_t n4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 f = __ldg(src + i);
    uint2 o;
    __nv_bfloat162 a = __floats2bfloat162_rn(f.x, f.y), b = __floats2bfloat162_rn(f.z, f.w);
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    dst[i] = o;
  }
}

int grid_for(int64_t work, int threads) {
  const int sms = device_sm_count();
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

template <typename T>
cudaError_t pyramid_dispatch(const void* k, const void* v, void* kp, void* vp, int64_t BH, int N, int d,
                             int levels, const size_t* off, cudaStream_t s) {
  const int G = 1 << (levels - 1);
  const int64_t work = 2 * BH * (N / G) * (d / Vec<T>::kN);
  const int grid = grid_for(work, 256);
  const T* kk = static_cast<const T*>(k);
  const T* vv = static_cast<const T*>(v);
  char* kpp = static_cast<char*>(kp);
  char* vpp = static_cast<char*>(vp);
  switch (G) {
    case 2: pyramid_kernel<T, 2><<<grid, 256, 0, s>>>(kk, vv, kpp, vpp, BH, N, d, off[1], 0, 0); break;
    case 4: pyramid_kernel<T, 4><<<grid, 256, 0, s>>>(kk, vv, kpp, vpp, BH, N, d, off[1], off[2], 0); break;
    case 8: pyramid_kernel<T, 8><<<grid, 256, 0, s>>>(kk, vv, kpp, vpp, BH, N, d, off[1], off[2], off[3]); break;
    default: return cudaSuccess;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pyramid(const void* k, const void* v, void* k_pyr, void* v_pyr, int64_t BH, int N,
                           int d, int levels, int elem, const size_t* level_off, cudaStream_t s) {
  if (levels <= 1) return cudaSuccess;
  if (elem == 2) return pyramid_dispatch<__nv_bfloat16>(k, v, k_pyr, v_pyr, BH, N, d, levels, level_off, s);
  return pyramid_dispatch<float>(k, v, k_pyr, v_pyr, BH, N, d, levels, level_off, s);
}

cudaError_t launch_blockcos(const void* k, float* out, int64_t BH, int N, int d, int block, int elem,
                            cudaStream_t s) {
  const int nkb = (N + block - 1) / block;
  dim3 grid(nkb, static_cast<unsigned>(BH));
  if (elem == 2) {
    const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(k);
    if (d == 128) blockcos_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(kk, out, N, block, nkb);
    else blockcos_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(kk, out, N, block, nkb);
  } else {
    const float* kk = static_cast<const float*>(k);
    if (d == 128) blockcos_kernel<float, 128><<<grid, 256, 0, s>>>(kk, out, N, block, nkb);
    else blockcos_kernel<float, 64><<<grid, 256, 0, s>>>(kk, out, N, block, nkb);
  }
  return cudaGetLastError();
}

cudaError_t launch_cast_bf16(const float* src, void* dst, int64_t n, cudaStream_t s) {
  const int64_t n4 = n / 4;   // every tensor here has d in {64, 128}: n % 4 == 0
  cast_kernel<<<grid_for(n4, 256), 256, 0, s>>>(reinterpret_cast<const float4*>(src),
                                                reinterpret_cast<uint2*>(dst), n4);
  return cudaGetLastError();
}

}  // namespace psa
