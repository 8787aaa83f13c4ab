// meankey.cu -- the mean-key block scorer of psa_make_mask (skill page
// "psa-pyramid-sparse-attention", Core Technique: a KV block is scored by
// the query against the mean of the block's keys; the query side is the
// query block's mean as well).  It reads Q and K once and does
// nQB * nKB * d multiply-adds per head, so it is bound by HBM bandwidth, not
// by the tensor cores.
//   blockmean_kernel      one CTA per (bh, block): fp64 mean of the block's
//                         valid tokens, one thread per channel.
//   meankey_score_kernel  one CTA per (bh, 8 query blocks): fp64 dot
//                         products of the query-block means against every
//                         key-block mean, written as log2-domain scores in
//                         the layout the select kernel reads, then the
//                         row's log-sum-exp over the visible key blocks.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"

namespace psa {
namespace {

constexpr int kRowsPerCta = 8;
constexpr int kScoreThreads = 256;

__device__ __forceinline__ double to_f64(float x) { return static_cast<double>(x); }
__device__ __forceinline__ double to_f64(__nv_bfloat16 x) { return static_cast<double>(__bfloat162float(x)); }

// x: [BH, N, d]; out: [BH, nb, d], or [BH, d, nb] when transpose (so that a
// warp reading one channel of consecutive blocks is coalesced).
template <typename T>
__global__ void blockmean_kernel(const T* __restrict__ x, double* __restrict__ out, int N, int d, int block, int nb,
                                 int transpose) {
  const int64_t bh = blockIdx.x / nb;
  const int J = static_cast<int>(blockIdx.x - bh * nb);
  const int t0 = J * block, t1 = min(t0 + block, N);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const T* p = x + (bh * N + t0) * d + c;
    double s = 0.0;
#pragma unroll 8
    for (int t = t0; t < t1; ++t, p += d) s += to_f64(*p);
    const double m = s / static_cast<double>(t1 - t0);
    if (transpose) out[(bh * d + c) * nb + J] = m;
    else out[(bh * nb + J) * d + c] = m;
  }
}

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kScoreThreads) meankey_score_kernel(const MeanKeyArgs a) {
  extern __shared__ double qs[];                       // [kRowsPerCta][d]
  __shared__ double red[kScoreThreads / 32][kRowsPerCta];
  __shared__ double rmax[kRowsPerCta], rsum[kRowsPerCta];
  const int groups = (a.nqb + kRowsPerCta - 1) / kRowsPerCta;
  const int bh = blockIdx.x / groups;
  const int I0 = (blockIdx.x - bh * groups) * kRowsPerCta;
  const int b = bh / a.Hq, h = bh - b * a.Hq;
  const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int nr = min(kRowsPerCta, a.nqb - I0);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kRowsPerCta * a.d; i += blockDim.x) {
    const int r = i / a.d, c = i - r * a.d;
    qs[i] = r < nr ? a.qmean[(static_cast<int64_t>(bh) * a.nqb + I0 + r) * a.d + c] : 0.0;
  }
  __syncthreads();
  const double* km = a.kmeanT + static_cast<int64_t>(hkv) * a.d * a.nkb;
  float* bl = a.blocklse + static_cast<int64_t>(bh) * a.nkb * a.nqb;

  // pass 1: scores (log2 domain) of every visible key block, row maxima
  double mx[kRowsPerCta];
#pragma unroll
  for (int r = 0; r < kRowsPerCta; ++r) mx[r] = -CUDART_INF;
  for (int J = threadIdx.x; J < a.nkb; J += blockDim.x) {
    double acc[kRowsPerCta];
#pragma unroll
    for (int r = 0; r < kRowsPerCta; ++r) acc[r] = 0.0;
    for (int c = 0; c < a.d; ++c) {
      const double kv = km[static_cast<int64_t>(c) * a.nkb + J];
#pragma unroll
      for (int r = 0; r < kRowsPerCta; ++r) acc[r] = fma(qs[r * a.d + c], kv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kRowsPerCta; ++r) {
      if (r < nr) {
        const int I = I0 + r;
        const bool vis = !a.causal || J <= I;
        const float z = vis ? static_cast<float>(acc[r] * a.scale_log2) : -CUDART_INF_F;
        bl[static_cast<int64_t>(J) * a.nqb + I] = z;
        if (vis) mx[r] = fmax(mx[r], static_cast<double>(z));
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerCta; ++r) {
    const double v = warp_max(mx[r]);
    if (lane == 0) red[wid][r] = v;
  }
  __syncthreads();
  if (threadIdx.x < kRowsPerCta) {
    double v = -CUDART_INF;
    for (int w = 0; w < kScoreThreads / 32; ++w) v = fmax(v, red[w][threadIdx.x]);
    rmax[threadIdx.x] = v;
  }
  __syncthreads();

  // pass 2: sum of 2^(z - max) over the scores this thread wrote
  double sm[kRowsPerCta];
#pragma unroll
  for (int r = 0; r < kRowsPerCta; ++r) sm[r] = 0.0;
  for (int J = threadIdx.x; J < a.nkb; J += blockDim.x) {
#pragma unroll
    for (int r = 0; r < kRowsPerCta; ++r) {
      if (r < nr) {
        const float z = bl[static_cast<int64_t>(J) * a.nqb + I0 + r];
        if (z != -CUDART_INF_F) sm[r] += exp2(static_cast<double>(z) - rmax[r]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerCta; ++r) {
    const double v = warp_sum(sm[r]);
    if (lane == 0) red[wid][r] = v;
  }
  __syncthreads();
  if (threadIdx.x < nr) {
    double v = 0.0;
    for (int w = 0; w < kScoreThreads / 32; ++w) v += red[w][threadIdx.x];
    const int64_t o = static_cast<int64_t>(bh) * a.nqb + I0 + threadIdx.x;
    a.rowlse[o] = static_cast<float>(rmax[threadIdx.x] + log2(v));
    a.rowlse[static_cast<int64_t>(a.BHq) * a.nqb + o] = -CUDART_INF_F;
  }
}

}  // namespace

cudaError_t launch_blockmean(const void* x, double* out, int64_t BH, int N, int d, int block, int elem,
                             bool transpose, cudaStream_t s) {
  const int nb = (N + block - 1) / block;
  const int64_t grid = BH * nb;
  const int threads = d < 128 ? d : 128;
  if (elem == 4)
    blockmean_kernel<float><<<static_cast<unsigned>(grid), threads, 0, s>>>(static_cast<const float*>(x), out, N, d,
                                                                              block, nb, transpose ? 1 : 0);
  else
    blockmean_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), threads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), out, N, d, block, nb, transpose ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_meankey_score(const MeanKeyArgs& a, cudaStream_t s) {
  const int groups = (a.nqb + kRowsPerCta - 1) / kRowsPerCta;
  const size_t smem = static_cast<size_t>(kRowsPerCta) * a.d * sizeof(double);
  meankey_score_kernel<<<static_cast<unsigned>(a.BHq) * groups, kScoreThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace psa
