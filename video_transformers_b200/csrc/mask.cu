// mask.cu -- stage 2 of the PSA forward path: the multi-level mask
// generator (summary article "PSA: Pyramid Sparse Attention ...", Method:
// importance of every query-block x KV-block pair, by sampled queries for
// generation and by antidiagonal scores for understanding; Results:
// threshold-based levels and a cosine condition for pooling).
//
// score_kernel   a tcgen05 GEMM of 128 score rows x 128 score columns per
//                tile (rows: sampled queries, or antidiagonal query groups;
//                columns: keys, or key groups), accumulated in TMEM, followed
//                by a per-(row, KV block) log-sum-exp in the epilogue warps.
//                Only the block LSEs and each row's total LSE leave the SM.
// select_kernel  one CTA per (b, h, query block): block masses from the
//                LSEs, a bitonic sort (mass descending, index ascending), an
//                fp64 exclusive scan, thresholds, forced rules.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kStages = 4;
constexpr int kChunkBytes = 128 * 128;        // 128 rows x 64 bf16
constexpr int kStageBytes = 2 * kChunkBytes;  // A chunk + B chunk
constexpr int kThreads = 192;                 // producer, MMA, 4 epilogue warps

struct ScoreShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ int kv_head_of(int bh, int Hq, int Hkv) {
  const int b = bh / Hq, h = bh - b * Hq;
  return b * Hkv + h / (Hq / Hkv);
}

template <int CPB>
__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const ScoreArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ScoreShared* sh = reinterpret_cast<ScoreShared*>(tiles + kStages * kStageBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_tiles = (a.rows + 127) / 128;
  const int col_tiles = (a.cols + 127) / 128;
  const int n_items = a.BHq * row_tiles;
  const int nk = (a.mode == 0 ? a.d / 64 : a.S * a.d / 64);
  const int kc_per_s = a.d / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(smem_u32(&sh->full[i]), 1); mbar_init(smem_u32(&sh->empty[i]), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&sh->s_full[i]), 1); mbar_init(smem_u32(&sh->s_empty[i]), 128); }
    mbar_init(smem_u32(&sh->drain), 1);
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&sh->tmem_base), 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;

  // number of column tiles a row tile visits (causal: up to its last row)
  auto tiles_for = [&](int r0) {
    if (!a.causal) return col_tiles;
    const int rlast = min(r0 + 127, a.rows - 1);
    const int pos = a.mode == 0 ? rlast * a.step : rlast;
    return min(col_tiles, pos / 128 + 1);
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
      uint32_t it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int bh = item / row_tiles, r0 = (item - bh * row_tiles) * 128;
        const int hkv = kv_head_of(bh, a.Hq, a.Hkv);
        const int nct = tiles_for(r0);
        for (int ct = 0; ct < nct && ok; ++ct) {
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int st = it % kStages;
            if (!bounded_wait(smem_u32(&sh->empty[st]), ((it / kStages) & 1) ^ 1, abort, a.status, 41, item, ct, kc, it)) { ok = false; break; }
            const uint32_t bar = smem_u32(&sh->full[st]);
            mbar_arrive_expect_tx(bar, kStageBytes);
            const uint32_t dA = smem_u32(tiles + st * kStageBytes);
            const uint32_t dB = dA + kChunkBytes;
            const int s = kc / kc_per_s, half = kc - s * kc_per_s;
            if (a.mode == 0) {
              tma_load_4d(dA, &mapA, bar, kc * 64, 0, r0, bh);
              tma_load_4d(dB, &mapB, bar, kc * 64, 0, ct * 128, hkv);
            } else {
              tma_load_4d(dA, &mapA, bar, half * 64, a.S - 1 - s, r0, bh);
              tma_load_4d(dB, &mapB, bar, half * 64, s, ct * 128, hkv);
            }
          }
        }
      }
      // drain: every armed stage must have landed before the CTA exits
      for (uint32_t st = 0; st < static_cast<uint32_t>(kStages); ++st) {
        if (it > st) drain_wait(smem_u32(&sh->full[st]), ((it - 1 - st) / kStages) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      uint32_t it = 0, t = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int bh = item / row_tiles, r0 = (item - bh * row_tiles) * 128;
        (void)bh;
        const int nct = tiles_for(r0);
        for (int ct = 0; ct < nct && ok; ++ct, ++t) {
          const int buf = t & 1;
          if (!bounded_wait(smem_u32(&sh->s_empty[buf]), ((t >> 1) & 1) ^ 1, abort, a.status, 42, item, ct, t, it)) { ok = false; break; }
          tc_fence_after();
          const uint32_t dS = tmem + buf * 128;
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int st = it % kStages;
            if (!bounded_wait(smem_u32(&sh->full[st]), (it / kStages) & 1, abort, a.status, 43, item, ct, kc, it)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sA = smem_u32(tiles + st * kStageBytes);
            const uint32_t sB = sA + kChunkBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              umma_ss(dS, sdesc_sw128(sA + 32 * k, 16, 1024), sdesc_sw128(sB + 32 * k, 16, 1024), idesc,
                      (kc | k) != 0);
            }
            umma_commit(smem_u32(&sh->empty[st]));
          }
          if (ok) umma_commit(smem_u32(&sh->s_full[buf]));
        }
      }
      umma_commit(smem_u32(&sh->drain));
      drain_wait(smem_u32(&sh->drain), 0, a.status);
    }
  } else {
    // ---------------- epilogue: per (row, block) log-sum-exp ----------------
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int lrow = q * 32 + lane;         // tile row owned by this thread
    constexpr int BPT = 128 / CPB;          // KV blocks per column tile
    uint32_t t = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int bh = item / row_tiles, r0 = (item - bh * row_tiles) * 128;
      const int r = r0 + lrow;
      const int pos = a.mode == 0 ? r * a.step : r;     // token (sampling) or group index
      const int nct = tiles_for(r0);
      float M = -CUDART_INF_F, Ssum = 0.f;
      for (int ct = 0; ct < nct; ++ct, ++t) {
        const int buf = t & 1;
        if (!warp_wait(smem_u32(&sh->s_full[buf]), (t >> 1) & 1, abort, a.status, 44, item, ct, t, 0)) { ok = false; break; }
        tc_fence_after();
        float z[128];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t raw[32];
          tmem_ld32(tmem + buf * 128 + c4 * 32 + (static_cast<uint32_t>(q * 32) << 16), raw);
#pragma unroll
          for (int j = 0; j < 32; ++j) z[c4 * 32 + j] = __uint_as_float(raw[j]) * a.scale_log2;
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->s_empty[buf]));
        const int c0 = ct * 128;
        const int climit = a.causal ? min(a.cols, pos + 1) : a.cols;   // valid columns: c < climit
#pragma unroll
        for (int bb = 0; bb < BPT; ++bb) {
          float m = -CUDART_INF_F;
#pragma unroll
          for (int j = 0; j < CPB; ++j) {
            const int c = c0 + bb * CPB + j;
            if (c < climit) m = fmaxf(m, z[bb * CPB + j]);
          }
          float s = 0.f;
          if (m != -CUDART_INF_F) {
#pragma unroll
            for (int j = 0; j < CPB; ++j) {
              const int c = c0 + bb * CPB + j;
              if (c < climit) s += fast_exp2(z[bb * CPB + j] - m);
            }
          }
          const float blse = m == -CUDART_INF_F ? -CUDART_INF_F : m + __log2f(s);
          const int J = (c0 / CPB) + bb;
          if (r < a.rows && J < a.nkb) a.blocklse[(static_cast<int64_t>(bh) * a.nkb + J) * a.rows + r] = blse;
          if (blse != -CUDART_INF_F) {
            const float Mn = fmaxf(M, blse);
            Ssum = Ssum * fast_exp2(M - Mn) + fast_exp2(blse - Mn);
            M = Mn;
          }
        }
      }
      if (!ok) break;
      // column tiles never visited (causal) hold no probability
      if (a.causal) {
        for (int J = nct * BPT; J < a.nkb; ++J)
          if (r < a.rows) a.blocklse[(static_cast<int64_t>(bh) * a.nkb + J) * a.rows + r] = -CUDART_INF_F;
      }
      if (r < a.rows) a.rowlse[static_cast<int64_t>(bh) * a.rows + r] = M == -CUDART_INF_F ? -CUDART_INF_F : M + __log2f(Ssum);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

// ----------------------------------------------------------------------------
// select: one CTA of 512 threads per (b, h, I)
// ----------------------------------------------------------------------------
constexpr int kSelThreads = 512;

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectArgs a) {
  __shared__ unsigned long long key[PSA_MAX_KV_BLOCKS];
  __shared__ double scan[PSA_MAX_KV_BLOCKS];
  __shared__ double warp_tot[kSelThreads / 32];
  const int row = blockIdx.x;                 // (b*Hq + h)*nqb + I
  const int bh = row / a.nqb, I = row - bh * a.nqb;
  const int b = bh / a.Hq, h = bh - b * a.Hq;
  const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  int P2 = 1;
  while (P2 < a.nkb) P2 <<= 1;

  // rows of the score that belong to query block I, and how many are valid
  const int rbeg = I * a.rows_per_block;
  int nvalid;
  if (a.mode == 0) {
    nvalid = 0;
    for (int s = 0; s < a.rows_per_block; ++s) nvalid += (static_cast<int64_t>(rbeg + s) * a.step < a.N);
  } else {
    nvalid = min(a.rows_per_block, a.rows - rbeg);
  }
  const float* rl = a.rowlse + static_cast<int64_t>(bh) * a.rows + rbeg;

  for (int J = threadIdx.x; J < P2; J += blockDim.x) {
    if (J < a.nkb) {
      const float* bl = a.blocklse + (static_cast<int64_t>(bh) * a.nkb + J) * a.rows + rbeg;
      double m = 0.0;
      for (int s = 0; s < nvalid; ++s) {
        const float x = bl[s];
        if (x != -CUDART_INF_F) m += exp2(static_cast<double>(x) - static_cast<double>(rl[s]));
      }
      const float mass = static_cast<float>(m / nvalid);
      if (a.mass_out) a.mass_out[static_cast<int64_t>(row) * a.nkb + J] = mass;
      scan[J] = mass;
      // ascending order of (descending mass, ascending J); mass >= 0 so its bits sort as uint
      key[J] = (static_cast<unsigned long long>(0xFFFFFFFFu - __float_as_uint(mass)) << 32) | static_cast<unsigned>(J);
    } else {
      key[J] = ~0ull;
    }
  }
  __syncthreads();
  // bitonic sort, ascending
  for (int k = 2; k <= P2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = key[i], y = key[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) { key[i] = y; key[ixj] = x; }
        }
      }
      __syncthreads();
    }
  }
  // exclusive prefix of the masses in sorted order, fp64; each thread owns a
  // contiguous run of ranks
  const int per = (P2 + blockDim.x - 1) / blockDim.x;
  const int k0 = threadIdx.x * per;
  double local = 0.0;
  for (int i = k0; i < min(k0 + per, a.nkb); ++i) local += scan[static_cast<int>(key[i] & 0xFFFFFFFFu)];
  // block exclusive scan of `local`
  double incl = local;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  double wbase = 0.0;
  for (int w = 0; w < wid; ++w) wbase += warp_tot[w];
  double C = wbase + incl - local;
  __syncthreads();
  for (int i = k0; i < min(k0 + per, a.nkb); ++i) {
    const int J = static_cast<int>(key[i] & 0xFFFFFFFFu);
    const double mJ = scan[J];
    int lev = 0;
    for (int l = 0; l < a.levels; ++l) lev += (static_cast<double>(a.thresholds[l]) <= C);
    int out = lev >= a.levels ? PSA_SKIP : lev;
    if (a.n_dense_prefix > 0 &&
        (static_cast<int64_t>(I) * a.block < a.n_dense_prefix || static_cast<int64_t>(J) * a.block < a.n_dense_prefix))
      out = 0;
    if (a.blockcos && a.cos_min > -2.f && out != PSA_SKIP && out >= 1 &&
        a.blockcos[static_cast<int64_t>(hkv) * a.nkb + J] < a.cos_min)
      out = 0;
    if (a.causal) {
      if (J > I) out = PSA_SKIP;
      else if (J == I) out = 0;
    }
    a.mask[static_cast<int64_t>(row) * a.nkb + J] = static_cast<uint8_t>(out);
    C += mJ;
  }
}

}  // namespace

cudaError_t launch_score(const CUtensorMap* mapA, const CUtensorMap* mapB, const ScoreArgs& a, int num_sms,
                         cudaStream_t s) {
  const int row_tiles = (a.rows + 127) / 128;
  const int n_items = a.BHq * row_tiles;
  const int grid = n_items < num_sms ? n_items : num_sms;
  const size_t smem = 1024 + kStages * kStageBytes + sizeof(ScoreShared);
  switch (a.cols_per_block) {
#define PSA_SCORE_CASE(CPB)                                                                       \
  case CPB: {                                                                                     \
    cudaError_t e = cudaFuncSetAttribute(score_kernel<CPB>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         static_cast<int>(smem));                                 \
    if (e != cudaSuccess) return e;                                                               \
    score_kernel<CPB><<<grid, kThreads, smem, s>>>(*mapA, *mapB, a);                              \
    break;                                                                                        \
  }
    PSA_SCORE_CASE(8)
    PSA_SCORE_CASE(16)
    PSA_SCORE_CASE(32)
    PSA_SCORE_CASE(64)
    PSA_SCORE_CASE(128)
#undef PSA_SCORE_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int rows = a.B * a.Hq * a.nqb;
  select_kernel<<<rows, kSelThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace psa
