// meankey.cu -- the mean-key block scorer of psa_make_mask (skill page
// "psa-pyramid-sparse-attention", Core Technique: a KV block is scored by
// the query against the mean of the block's keys; the query side is the
// query block's mean as well).  It reads Q and K once and does
// nQB * nKB * d multiply-adds per head, so it is bound by HBM bandwidth, not
// by the tensor cores.
//   blockmean_kernel       one CTA per (bh, block): fp64 mean of the block's
//                          valid tokens, one thread per channel, written
//                          channel-major.
//   meankey_logits_kernel  a 64 x 64 tile of (query block, key block) pairs
//                          per CTA: fp64 dot products of the means, written
//                          as log2-domain scores in the layout the select
//                          kernel reads.
//   meankey_lse_kernel     the row log-sum-exp over the visible key blocks.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"

namespace psa {
namespace {

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

// Logits of a 64 x 64 tile of (query block I, key block J) pairs of one head
// (fp64, 256 threads, 4 x 4 pairs per thread): thread (ty, tx) owns
// I = I0 + tx + 16u and J = J0 + ty + 16v, so stores of one J are
// contiguous in I.  The means arrive channel-major ([bh][c][block]).
constexpr int kTile = 64;
constexpr int kChan = 32;

__global__ void __launch_bounds__(256) meankey_logits_kernel(const MeanKeyArgs a) {
  __shared__ double qt[kChan][kTile];
  __shared__ double kt[kChan][kTile];
  const int bh = blockIdx.y;
  const int tiles_i = (a.nqb + kTile - 1) / kTile;
  const int I0 = (blockIdx.x % tiles_i) * kTile, J0 = (blockIdx.x / tiles_i) * kTile;
  const int b = bh / a.Hq, h = bh - b * a.Hq;
  const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const double* qm = a.qmean + static_cast<int64_t>(bh) * a.d * a.nqb;
  const double* km = a.kmeanT + static_cast<int64_t>(hkv) * a.d * a.nkb;
  double acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
  for (int c0 = 0; c0 < a.d; c0 += kChan) {
    __syncthreads();
    for (int i = threadIdx.x; i < kChan * kTile; i += 256) {
      const int c = i / kTile, x = i - c * kTile;
      const bool cin = c0 + c < a.d;
      qt[c][x] = cin && I0 + x < a.nqb ? qm[static_cast<int64_t>(c0 + c) * a.nqb + I0 + x] : 0.0;
      kt[c][x] = cin && J0 + x < a.nkb ? km[static_cast<int64_t>(c0 + c) * a.nkb + J0 + x] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kChan; ++c) {
      double qv[4], kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) qv[u] = qt[c][tx + 16 * u];
#pragma unroll
      for (int v = 0; v < 4; ++v) kv[v] = kt[c][ty + 16 * v];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(qv[u], kv[v], acc[u][v]);
    }
  }
  float* bl = a.blocklse + static_cast<int64_t>(bh) * a.nkb * a.nqb;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int J = J0 + ty + 16 * v;
    if (J >= a.nkb) continue;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int I = I0 + tx + 16 * u;
      if (I >= a.nqb) continue;
      const bool vis = !a.causal || J <= I;
      bl[static_cast<int64_t>(J) * a.nqb + I] = vis ? static_cast<float>(acc[u][v] * a.scale_log2) : -CUDART_INF_F;
    }
  }
}

// Row log-sum-exp (log2 domain, fp64) over the visible key blocks, one
// thread per (bh, I); a warp reads one J of 32 consecutive rows at a time.
__global__ void __launch_bounds__(256) meankey_lse_kernel(const MeanKeyArgs a) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(a.BHq) * a.nqb) return;
  const int64_t bh = t / a.nqb;
  const int I = static_cast<int>(t - bh * a.nqb);
  const float* bl = a.blocklse + bh * a.nkb * a.nqb + I;
  const int nj = a.causal ? min(I + 1, a.nkb) : a.nkb;
  double mx = -CUDART_INF;
  for (int J = 0; J < nj; ++J) mx = fmax(mx, static_cast<double>(bl[static_cast<int64_t>(J) * a.nqb]));
  double sm = 0.0;
  for (int J = 0; J < nj; ++J) sm += exp2(static_cast<double>(bl[static_cast<int64_t>(J) * a.nqb]) - mx);
  a.rowlse[t] = static_cast<float>(mx + log2(sm));
  a.rowlse[static_cast<int64_t>(a.BHq) * a.nqb + t] = -CUDART_INF_F;
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
  const int tiles = ((a.nqb + kTile - 1) / kTile) * ((a.nkb + kTile - 1) / kTile);
  meankey_logits_kernel<<<dim3(tiles, a.BHq), 256, 0, s>>>(a);
  const int64_t rows = static_cast<int64_t>(a.BHq) * a.nqb;
  meankey_lse_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace psa
