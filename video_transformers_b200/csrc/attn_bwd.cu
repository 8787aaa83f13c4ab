// attn_bwd.cu -- gradients of adaptive pyramid attention with respect to Q,
// K and V (news review "[Paper] PSA ...", Methodology 4: the model is
// trained end to end through the pooled attention; summary article
// "PSA: Pyramid Sparse Attention ...", Results: PSA is paired with
// distillation).  The pages give no backward pass; it is the derivative of
// the forward's definition, the mask being a fixed selection: for query i,
// pooled key p of level l, z = sm_scale q.K^l[p] + l ln 2, P = exp(z - lse),
//   dP = dO.V^l[p],  D = dO.O,  dZ = P (dP - D),
//   dQ = sm_scale sum_p dZ K^l[p],  dK^l[p] = sm_scale sum_i dZ q_i,
//   dV^l[p] = sum_i P dO_i,
// then through the pooling of each level: token t of level 0 receives
// dK^l[t >> l] / 2^l from every level l.
//
// bwd_prep_kernel   D = dO.O and lse in log2 units, padded to 128-row tiles.
// dq_kernel         query-major, on the forward's tile plan: per 64-row KV
//                   sub-tile S = Q K^T and dP = dO V^T (tcgen05, TMEM), dS as
//                   bf16 back into TMEM, dQ += dS K (A from TMEM).
// tplan_*           the transposed plan: for every 128-row tile of one
//                   pyramid level of one KV head, the query tiles that use it.
// dkv_kernel        KV-major: per (KV tile, query tile) S^T = K Q^T and
//                   dP^T = V dO^T (M = 128 KV rows, N = 64 query rows per
//                   half), P^T and dS^T as bf16 into TMEM, dV += P^T dO and
//                   dK += dS^T Q accumulated in TMEM over all query tiles.
// pool_bwd_kernel   the level gradients folded into dK, dV (HBM-bound).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ----------------------------------------------------------------------------
// D and lse2, padded
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2p,
                                                       float* __restrict__ dp, int64_t BHq, int N, int d, int n_qt) {
  const int64_t rows_p = static_cast<int64_t>(n_qt) * 128;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= BHq * rows_p) return;
  const int64_t bh = warp / rows_p;
  const int i = static_cast<int>(warp - bh * rows_p);
  float acc = 0.f;
  if (i < N) {
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(out + (bh * N + i) * d);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(dout + (bh * N + i) * d);
    for (int c = lane; c < d / 2; c += 32) {
      const float2 x = __bfloat1622float2(o2[c]);
      const float2 y = __bfloat1622float2(g2[c]);
      acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  }
  if (lane == 0) {
    // rows past N, and rows that saw no key (lse = -inf, output 0), get
    // lse2 = +inf: every probability of theirs is then exactly 0
    const float l = i < N ? lse[bh * N + i] : -CUDART_INF_F;
    lse2p[warp] = l == -CUDART_INF_F ? CUDART_INF_F : l * kLog2e;
    dp[warp] = i < N ? acc : 0.f;
  }
}

// ----------------------------------------------------------------------------
// pooling backward: one thread per 4 channels of one token
// ----------------------------------------------------------------------------
struct LevelOff {
  int64_t off[4];
};

__global__ void __launch_bounds__(256) pool_bwd_kernel(const float* __restrict__ gl, const LevelOff lo,
                                                       __nv_bfloat16* __restrict__ out, int64_t BHkv, int N, int d,
                                                       int levels) {
  const int d4 = d / 4;
  const int64_t total = BHkv * N * d4;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = x / d4;
    const int c4 = static_cast<int>(x - row * d4);
    const int64_t bh = row / N;
    const int t = static_cast<int>(row - bh * N);
    float4 acc = *reinterpret_cast<const float4*>(gl + lo.off[0] + row * d + 4 * c4);
    for (int l = 1; l < levels; ++l) {
      const int Nl = N >> l;
      const float w = 1.0f / static_cast<float>(1 << l);
      const float4 g = *reinterpret_cast<const float4*>(gl + lo.off[l] + (bh * Nl + (t >> l)) * d + 4 * c4);
      acc.x = fmaf(g.x, w, acc.x);
      acc.y = fmaf(g.y, w, acc.y);
      acc.z = fmaf(g.z, w, acc.z);
      acc.w = fmaf(g.w, w, acc.w);
    }
    __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y), b = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(out + row * d + 4 * c4) = o;
  }
}

// ----------------------------------------------------------------------------
// transposed plan
// ----------------------------------------------------------------------------
struct TItem {
  int l, b, hkv, t;     // level, batch, KV head (within the batch), tile
};

__device__ __forceinline__ TItem titem(const int* level_base, const int* level_tiles, int Hkv, int item) {
  TItem r;
  r.l = 0;
  while (item >= level_base[r.l + 1]) ++r.l;
  const int local = item - level_base[r.l];
  const int bhkv = local / level_tiles[r.l];
  r.t = local - bhkv * level_tiles[r.l];
  r.b = bhkv / Hkv;
  r.hkv = bhkv - r.b * Hkv;
  return r;
}

// Bit 2 jb + hf: block jb of the item's tile is at level l for query half hf
// of query tile tq of head h, and some of its pooled tokens are visible.
__device__ __forceinline__ unsigned entry_bits(const TPlanArgs& a, const TItem& it, int h, int tq) {
  const int rows_blk = a.block >> it.l;
  const int nJ = 128 / rows_blk;
  const int J0 = it.t * nJ;
  const uint8_t* m = a.mask + static_cast<int64_t>(it.b * a.Hq + h) * a.nqb * a.nkb;
  unsigned bits = 0;
  const int halves = a.block == 128 ? 1 : 2;
  for (int hf = 0; hf < halves; ++hf) {
    const int I = a.block == 128 ? tq : 2 * tq + hf;
    if (I >= a.nqb) continue;
    const int imax = min((I + 1) * a.block, a.N) - 1;
    const uint8_t* row = m + static_cast<int64_t>(I) * a.nkb;
    for (int jb = 0; jb < nJ; ++jb) {
      const int J = J0 + jb;
      if (J >= a.nkb) break;
      if (row[J] == it.l && (!a.causal || J * a.block + (1 << it.l) - 1 <= imax)) bits |= 1u << (2 * jb + hf);
    }
  }
  if (a.block == 128) bits |= bits << 1;     // both query halves of a 128-token block agree
  return bits;
}

__global__ void tplan_count(const TPlanArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= a.n_items) return;
  const TItem it = titem(a.level_base, a.level_tiles, a.Hkv, warp);
  const int grp = a.Hq / a.Hkv;
  const int n = grp * a.n_qtiles;
  int c = 0;
  for (int x = lane; x < n; x += 32) {
    const int hl = x / a.n_qtiles, tq = x - hl * a.n_qtiles;
    c += entry_bits(a, it, it.hkv * grp + hl, tq) != 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) a.item_cnt[warp] = c;
}

__global__ void __launch_bounds__(1024) tplan_scan(const TPlanArgs a) {
  __shared__ long long wsum[32];
  __shared__ long long carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < a.n_items; base += blockDim.x) {
    const int i = base + tid;
    const long long v = i < a.n_items ? a.item_cnt[i] : 0;
    long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    long long w = 0;
    for (int x = 0; x < wid; ++x) w += wsum[x];
    const long long off = carry + w + inc - v;
    if (i < a.n_items) a.item_off[i] = static_cast<int>(off);
    __syncthreads();
    if (tid == blockDim.x - 1) carry = off + v;
    __syncthreads();
  }
  if (tid == 0) a.item_off[a.n_items] = static_cast<int>(carry);
}

__global__ void tplan_fill(const TPlanArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= a.n_items) return;
  const TItem it = titem(a.level_base, a.level_tiles, a.Hkv, warp);
  const int grp = a.Hq / a.Hkv;
  const int n = grp * a.n_qtiles;
  int k = a.item_off[warp];
  for (int x0 = 0; x0 < n; x0 += 32) {
    const int x = x0 + lane;
    unsigned bits = 0;
    if (x < n) {
      const int hl = x / a.n_qtiles, tq = x - hl * a.n_qtiles;
      bits = entry_bits(a, it, it.hkv * grp + hl, tq);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, bits != 0);
    if (bits) {
      const int idx = k + __popc(bal & ((1u << lane) - 1u));
      a.entry_qt[idx] = x;
      a.entry_mask[idx] = bits;
    }
    k += __popc(bal);
  }
}

}  // namespace

cudaError_t launch_bwd_prep(const void* out, const void* dout, const float* lse, float* lse2p, float* dp,
                            int64_t BHq, int N, int d, int n_qtiles, cudaStream_t s) {
  const int64_t rows = BHq * n_qtiles * 128;
  const int64_t grid = (rows * 32 + 255) / 256;
  bwd_prep_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(out),
                                                              static_cast<const __nv_bfloat16*>(dout), lse, lse2p,
                                                              dp, BHq, N, d, n_qtiles);
  return cudaGetLastError();
}

cudaError_t launch_pool_bwd(const float* gl, const int64_t* level_off, void* out, int64_t BHkv, int N, int d,
                            int levels, cudaStream_t s) {
  LevelOff lo;
  for (int l = 0; l < 4; ++l) lo.off[l] = l < levels ? level_off[l] : 0;
  const int64_t total = BHkv * N * (d / 4);
  const int64_t want = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
  const int grid = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
  pool_bwd_kernel<<<grid, 256, 0, s>>>(gl, lo, static_cast<__nv_bfloat16*>(out), BHkv, N, d, levels);
  return cudaGetLastError();
}

cudaError_t launch_tplan(const TPlanArgs& a, cudaStream_t s) {
  const int warps_per_cta = 8;
  const int grid = (a.n_items + warps_per_cta - 1) / warps_per_cta;
  tplan_count<<<grid, 32 * warps_per_cta, 0, s>>>(a);
  tplan_scan<<<1, 1024, 0, s>>>(a);
  tplan_fill<<<grid, 32 * warps_per_cta, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace psa
