// mask.cu -- stage 2 of the PSA forward path: the multi-level mask
// generator (summary article "PSA: Pyramid Sparse Attention ...", Method:
// importance of every query-block x KV-block pair, by sampled queries for
// generation and by antidiagonal scores for understanding; Results:
// threshold-based levels and a cosine condition for pooling).
//
// score_kernel   a tcgen05 GEMM of 128 score rows x 128 score columns per
//                tile (rows: sampled queries, or antidiagonal query groups;
//                columns: keys, or key groups), accumulated in TMEM, followed
//                by a per-(row, KV block) log-sum-exp in two epilogue
//                warpgroups that take alternate column tiles.  Only the block
//                LSEs and each row's LSE (one partial per warpgroup) leave
//                the SM.  Used for the antidiagonal score and for sampling at
//                d = 64.
// score2_kernel  the sampling score at d = 128: two row tiles share every K
//                tile, epilogue warpgroup x owns row tile x, and a work item
//                covers a quarter of the column tiles (one row-LSE partial
//                per quarter).
// select_bucket_kernel  one warp per (b, h, query block), up to 1024 key
//                blocks: the same levels as select_kernel without a sort --
//                a histogram of the masses in 256 buckets and its scan give
//                every block's level, except in the few buckets a threshold
//                falls into, whose blocks count their exact prefix (or rank).
// select_kernel  (more than 1024 key blocks) one CTA per (b, h, query
//                block): block masses from the LSEs, a bitonic sort (mass
//                descending, index ascending), an fp64 exclusive scan, levels
//                by that prefix (or by rank for the quantile policy), forced
//                rules.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "exp2_poly.h"
#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kThreads = 320;                 // producer, MMA, two epilogue warpgroups
constexpr int kChunk = 128 * 128;             // 128 rows x 64 bf16: one 128-byte-swizzled chunk
constexpr int kRegionChunks = 8;              // 128 KB of staging
// Sampling: A (the sampled query rows, <= 2 chunks) stays resident in chunks
// [0, 2) for all column tiles of a row tile; K chunks stream through a ring
// in chunks [2, 8).  Antidiagonal: A and B both stream, one (A, B) chunk
// pair per stage, four stages.
constexpr int kSampleStages = 6;
constexpr int kAntiStages = 4;

struct ScoreShared {
  uint64_t a_full, a_empty;
  uint64_t full[kSampleStages], empty[kSampleStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ int kv_head_of(int bh, int Hq, int Hkv) {
  const int b = bh / Hq, h = bh - b * Hq;
  return b * Hkv + h / (Hq / Hkv);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Of every 8 column pairs of a block, this many take their exponential on
// the FMA pipe (exp2_fma2_d5) instead of the special-function unit.
#ifndef PSA_SCORE_POLY
#define PSA_SCORE_POLY 0
#endif
constexpr int kScorePoly = PSA_SCORE_POLY;


// 2^x for two lanes at once on the FMA pipe, x <= 20, relative error about
// 2.4e-7: Cody-Waite split x = n + f with n = round(x) (adding 1.5 * 2^23
// rounds to an integer in the low mantissa bits) and f in [-1/2, 1/2]; 2^f
// from the degree-5 Remez polynomial of exp2_poly.h; 2^n added to the
// exponent field as an integer.  Inputs below -126 are clamped there (the
// result is then about 2^-126 instead of 0, far below one part in 10^30 of
// a block sum, whose largest term is 1).
__device__ __forceinline__ float2 exp2_fma2_d5(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
  const float2 n = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(kExp2Poly5_5, kExp2Poly5_5), f, make_float2(kExp2Poly5_4, kExp2Poly5_4));
  p = __ffma2_rn(p, f, make_float2(kExp2Poly5_3, kExp2Poly5_3));
  p = __ffma2_rn(p, f, make_float2(kExp2Poly5_2, kExp2Poly5_2));
  p = __ffma2_rn(p, f, make_float2(kExp2Poly5_1, kExp2Poly5_1));
  p = __ffma2_rn(p, f, make_float2(kExp2Poly5_0, kExp2Poly5_0));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// log2-domain log-sum-exp of CPB consecutive scores s[0..CPB) (already
// masked to -inf where invalid when MASKED), scaled by sc.
template <int CPB, bool MASKED>
__device__ __forceinline__ float block_lse(const float* s, float sc) {
  static_assert(CPB % 4 == 0 && CPB >= 8, "block width");
  float x[4] = {s[0], s[1], s[2], s[3]};
  constexpr int J8 = 4 + (CPB - 4) / 8 * 8;     // end of the 8-wide steps
#pragma unroll
  for (int j = 4; j < J8; j += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = fmax3(x[u], s[j + u], s[j + 4 + u]);
  }
#pragma unroll
  for (int j = J8; j < CPB; j += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = fmaxf(x[u], s[j + u]);
  }
  const float mraw = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  if (MASKED && mraw == -CUDART_INF_F) return -CUDART_INF_F;
  const float mb = mraw * sc;
  const float2 sc2 = make_float2(sc, sc), off = make_float2(-mb, -mb);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int j = 0; j < CPB; j += 2) {
    const float2 z = __ffma2_rn(make_float2(s[j], s[j + 1]), sc2, off);
    const float2 e = ((j >> 1) & 7) < kScorePoly ? exp2_fma2_d5(z) : make_float2(fast_exp2(z.x), fast_exp2(z.y));
    acc[(j >> 1) & 1] = __fadd2_rn(acc[(j >> 1) & 1], e);
  }
  const float2 t = __fadd2_rn(acc[0], acc[1]);
  return mb + __log2f(t.x + t.y);
}

template <int CPB>
__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const ScoreArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ScoreShared* sh = reinterpret_cast<ScoreShared*>(tiles + kRegionChunks * kChunk);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_tiles = (a.rows + 127) / 128;
  const int col_tiles = (a.cols + 127) / 128;
  const int n_items = a.BHq * row_tiles;
  const bool sampling = a.mode == 0;
  const int nk = sampling ? a.d / 64 : a.S * a.d / 64;   // 64-channel chunks per column tile
  const int kc_per_s = a.d / 64;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->a_full), 1);
    mbar_init(smem_u32(&sh->a_empty), 1);
    for (int i = 0; i < kSampleStages; ++i) { mbar_init(smem_u32(&sh->full[i]), 1); mbar_init(smem_u32(&sh->empty[i]), 1); }
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
    const int pos = sampling ? rlast * a.step : rlast;
    return min(col_tiles, pos / 128 + 1);
  };
  const int nst = sampling ? kSampleStages : kAntiStages;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
      uint32_t it = 0, icnt = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++icnt) {
        const int bh = item / row_tiles, r0 = (item - bh * row_tiles) * 128;
        const int hkv = kv_head_of(bh, a.Hq, a.Hkv);
        const int nct = tiles_for(r0);
        if (sampling) {
          if (!bounded_wait(smem_u32(&sh->a_empty), (icnt & 1) ^ 1, abort, a.status, 45, item, 0, 0, icnt)) { ok = false; break; }
          mbar_arrive_expect_tx(smem_u32(&sh->a_full), nk * kChunk);
          for (int kc = 0; kc < nk; ++kc)
            tma_load_4d(smem_u32(tiles + kc * kChunk), &mapA, smem_u32(&sh->a_full), kc * 64, 0, r0, bh);
        }
        for (int ct = 0; ct < nct && ok; ++ct) {
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int st = it % nst;
            if (!bounded_wait(smem_u32(&sh->empty[st]), ((it / nst) & 1) ^ 1, abort, a.status, 41, item, ct, kc, it)) { ok = false; break; }
            const uint32_t bar = smem_u32(&sh->full[st]);
            if (sampling) {
              mbar_arrive_expect_tx(bar, kChunk);
              tma_load_4d(smem_u32(tiles + (2 + st) * kChunk), &mapB, bar, kc * 64, 0, ct * 128, hkv);
            } else {
              const int s = kc / kc_per_s, half = kc - s * kc_per_s;
              mbar_arrive_expect_tx(bar, 2 * kChunk);
              tma_load_4d(smem_u32(tiles + (2 * st) * kChunk), &mapA, bar, half * 64, a.S - 1 - s, r0, bh);
              tma_load_4d(smem_u32(tiles + (2 * st + 1) * kChunk), &mapB, bar, half * 64, s, ct * 128, hkv);
            }
          }
        }
      }
      // drain: every armed stage must have landed before the CTA exits
      for (uint32_t st = 0; st < static_cast<uint32_t>(nst); ++st)
        if (it > st) drain_wait(smem_u32(&sh->full[st]), ((it - 1 - st) / nst) & 1, a.status);
      if (sampling && icnt > 0) drain_wait(smem_u32(&sh->a_full), (icnt - 1) & 1, a.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      const uint64_t d0 = sdesc_sw128(smem_u32(tiles), 16, 1024);
      uint32_t it = 0, t = 0, icnt = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++icnt) {
        const int bh = item / row_tiles, r0 = (item - bh * row_tiles) * 128;
        (void)bh;
        const int nct = tiles_for(r0);
        if (sampling) {
          if (!bounded_wait(smem_u32(&sh->a_full), icnt & 1, abort, a.status, 46, item, 0, 0, icnt)) { ok = false; break; }
          tc_fence_after();
        }
        for (int ct = 0; ct < nct && ok; ++ct, ++t) {
          const int buf = t & 1;
          if (!bounded_wait(smem_u32(&sh->s_empty[buf]), ((t >> 1) & 1) ^ 1, abort, a.status, 42, item, ct, t, it)) { ok = false; break; }
          tc_fence_after();
          const uint32_t dS = tmem + buf * 128;
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int st = it % nst;
            if (!bounded_wait(smem_u32(&sh->full[st]), (it / nst) & 1, abort, a.status, 43, item, ct, kc, it)) { ok = false; break; }
            tc_fence_after();
            const int ca = sampling ? kc : 2 * st;
            const int cb = sampling ? 2 + st : 2 * st + 1;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_ss(dS, d0 + ((ca * kChunk + 32 * k) >> 4), d0 + ((cb * kChunk + 32 * k) >> 4), idesc, (kc | k) != 0);
            umma_commit(smem_u32(&sh->empty[st]));
          }
          if (!ok) break;
          umma_commit(smem_u32(&sh->s_full[buf]));
          if (sampling && ct + 1 == nct) umma_commit(smem_u32(&sh->a_empty));
        }
      }
      umma_commit(smem_u32(&sh->drain));
      drain_wait(smem_u32(&sh->drain), 0, a.status);
    }
  } else {
    // ---------- epilogue: two warpgroups take alternate column tiles ----------
    const int wg = (warp - 2) >> 2;         // 0 or 1: the S buffer this group reads
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int lrow = q * 32 + lane;         // tile row owned by this thread
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    constexpr int BPT = 128 / CPB;          // KV blocks per column tile
    uint32_t t = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int bh = item / row_tiles, r0 = (item - bh * row_tiles) * 128;
      const int r = r0 + lrow;
      const int pos = sampling ? r * a.step : r;     // token (sampling) or group index
      const int nct = tiles_for(r0);
      const int climit = a.causal ? min(a.cols, pos + 1) : a.cols;   // valid columns: c < climit
      float M = -CUDART_INF_F, Ssum = 0.f;
      float* bl = a.blocklse + static_cast<int64_t>(bh) * a.nkb * a.rows + r;
      for (int ct = 0; ct < nct; ++ct, ++t) {
        if ((t & 1) != static_cast<uint32_t>(wg)) continue;
        if (!warp_wait(smem_u32(&sh->s_full[wg]), (t >> 1) & 1, abort, a.status, 44, item, ct, t, wg)) { ok = false; break; }
        tc_fence_after();
        uint32_t raw[128];
        tmem_ld128(tmem + wg * 128 + lane_off, raw);
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->s_empty[wg]));
        float* z = reinterpret_cast<float*>(raw);
        const int c0 = ct * 128;
        float blse[BPT];
        if (c0 + 128 <= climit) {
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) blse[bb] = block_lse<CPB, false>(z + bb * CPB, a.scale_log2);
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) z[c] = c0 + c < climit ? z[c] : -CUDART_INF_F;
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) blse[bb] = block_lse<CPB, true>(z + bb * CPB, a.scale_log2);
        }
        float mt = blse[0];
#pragma unroll
        for (int bb = 1; bb < BPT; ++bb) mt = fmaxf(mt, blse[bb]);
        if (mt != -CUDART_INF_F) {
          const float Mn = fmaxf(M, mt);
          float add = 0.f;
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) add += fast_exp2(blse[bb] - Mn);
          Ssum = Ssum * fast_exp2(M - Mn) + add;
          M = Mn;
        }
        if (r < a.rows) {
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) {
            const int J = ct * BPT + bb;
            if (J < a.nkb) bl[static_cast<int64_t>(J) * a.rows] = blse[bb];
          }
        }
      }
      if (!ok) break;
      if (r < a.rows) {
        // column tiles never visited (causal) hold no probability
        if (wg == 0) {
          for (int J = nct * BPT; J < a.nkb; ++J) bl[static_cast<int64_t>(J) * a.rows] = -CUDART_INF_F;
        }
        a.rowlse[(static_cast<int64_t>(wg) * a.BHq + bh) * a.rows + r] =
            M == -CUDART_INF_F ? -CUDART_INF_F : M + __log2f(Ssum);
      }
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
// score2_kernel: the sampling score with two row tiles per work item, so
// every K tile brought into shared memory serves 256 sampled rows instead of
// 128 (half the K traffic per flop).  A work item is (head, row-tile pair,
// part e of kScore2Parts of the column tiles); the two sampled-query tiles
// stay resident; TMEM holds two S buffers per row tile (512 columns);
// epilogue warpgroup x owns row tile x and writes row-LSE partial e.  Used for
// d = 128, where it halves the K traffic that bounds the one-row-tile
// kernel; at d = 64 (half the MMA work per tile) it measured slower.
// ----------------------------------------------------------------------------
constexpr int kRegion2 = 12;        // 192 KB: 2 * (d/64) resident A chunks + the K ring
constexpr int kMaxStages2 = 10;

struct Score2Shared {
  uint64_t a_full, a_empty;
  uint64_t full[kMaxStages2], empty[kMaxStages2];
  uint64_t s_full[2], s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int CPB>
__global__ void __launch_bounds__(kThreads, 1)
    score2_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                  const ScoreArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Score2Shared* sh = reinterpret_cast<Score2Shared*>(tiles + kRegion2 * kChunk);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_tiles = (a.rows + 127) / 128;
  const int pairs = (row_tiles + 1) / 2;
  const int col_tiles = (a.cols + 127) / 128;
  // item = (bh, row-tile pair, column part): the parts of a pair's column
  // sweep are separate items (finer work, a shorter last wave of the
  // persistent grid); part e writes row-LSE partial e
  const int n_items = a.BHq * pairs * kScore2Parts;
  const int nk = a.d / 64;                 // 64-channel chunks per tile
  const int nst = kRegion2 - 2 * nk;       // K ring stages (8 for d = 128, 10 for d = 64)

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->a_full), 1);
    mbar_init(smem_u32(&sh->a_empty), 1);
    for (int i = 0; i < kMaxStages2; ++i) { mbar_init(smem_u32(&sh->full[i]), 1); mbar_init(smem_u32(&sh->empty[i]), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&sh->s_full[i]), 1); mbar_init(smem_u32(&sh->s_empty[i]), 256); }
    mbar_init(smem_u32(&sh->drain), 1);
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&sh->tmem_base), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;

  // row tiles of a pair that exist, and the column tiles the pair visits
  // (causal: up to the last row of its last tile)
  auto n_rt = [&](int p) { return 2 * p + 1 < row_tiles ? 2 : 1; };
  auto tiles_for = [&](int p) {
    if (!a.causal) return col_tiles;
    const int rlast = min((2 * p + n_rt(p)) * 128 - 1, a.rows - 1);
    return min(col_tiles, rlast * a.step / 128 + 1);
  };
  // column tiles [lo, hi) of item part e (possibly empty for short causal rows)
  auto range_of = [&](int p, int e, int& lo, int& hi) {
    const int nct = tiles_for(p);
    lo = nct * e / kScore2Parts;
    hi = nct * (e + 1) / kScore2Parts;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
      uint32_t it = 0, icnt = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int e = item % kScore2Parts, bh = (item / kScore2Parts) / pairs, p = item / kScore2Parts - bh * pairs;
        const int hkv = kv_head_of(bh, a.Hq, a.Hkv);
        const int nrt = n_rt(p);
        int lo, hi;
        range_of(p, e, lo, hi);
        if (hi == lo) continue;
        if (!bounded_wait(smem_u32(&sh->a_empty), (icnt & 1) ^ 1, abort, a.status, 45, item, 0, 0, icnt)) { ok = false; break; }
        ++icnt;
        mbar_arrive_expect_tx(smem_u32(&sh->a_full), nrt * nk * kChunk);
        for (int x = 0; x < nrt; ++x)
          for (int kc = 0; kc < nk; ++kc)
            tma_load_4d(smem_u32(tiles + (x * nk + kc) * kChunk), &mapA, smem_u32(&sh->a_full), kc * 64, 0,
                        (2 * p + x) * 128, bh);
        for (int ct = lo; ct < hi && ok; ++ct) {
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int st = it % nst;
            if (!bounded_wait(smem_u32(&sh->empty[st]), ((it / nst) & 1) ^ 1, abort, a.status, 41, item, ct, kc, it)) { ok = false; break; }
            const uint32_t bar = smem_u32(&sh->full[st]);
            mbar_arrive_expect_tx(bar, kChunk);
            tma_load_4d(smem_u32(tiles + (2 * nk + st) * kChunk), &mapB, bar, kc * 64, 0, ct * 128, hkv);
          }
        }
      }
      for (uint32_t st = 0; st < static_cast<uint32_t>(nst); ++st)
        if (it > st) drain_wait(smem_u32(&sh->full[st]), ((it - 1 - st) / nst) & 1, a.status);
      if (icnt > 0) drain_wait(smem_u32(&sh->a_full), (icnt - 1) & 1, a.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      const uint64_t d0 = sdesc_sw128(smem_u32(tiles), 16, 1024);
      uint32_t it = 0, t = 0, icnt = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int e = item % kScore2Parts, bh = (item / kScore2Parts) / pairs, p = item / kScore2Parts - bh * pairs;
        (void)bh;
        const int nrt = n_rt(p);
        int lo, hi;
        range_of(p, e, lo, hi);
        if (hi == lo) continue;
        if (!bounded_wait(smem_u32(&sh->a_full), icnt & 1, abort, a.status, 46, item, 0, 0, icnt)) { ok = false; break; }
        ++icnt;
        tc_fence_after();
        for (int ct = lo; ct < hi && ok; ++ct, ++t) {
          const int b = t & 1;
          if (!bounded_wait(smem_u32(&sh->s_empty[b]), ((t >> 1) & 1) ^ 1, abort, a.status, 42, item, ct, t, it)) { ok = false; break; }
          tc_fence_after();
          for (int kc = 0; kc < nk; ++kc, ++it) {
            const int st = it % nst;
            if (!bounded_wait(smem_u32(&sh->full[st]), (it / nst) & 1, abort, a.status, 43, item, ct, kc, it)) { ok = false; break; }
            tc_fence_after();
            for (int x = 0; x < nrt; ++x) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_ss(tmem + x * 256 + b * 128, d0 + (((x * nk + kc) * kChunk + 32 * k) >> 4),
                        d0 + (((2 * nk + st) * kChunk + 32 * k) >> 4), idesc, (kc | k) != 0);
            }
            umma_commit(smem_u32(&sh->empty[st]));
          }
          if (!ok) break;
          umma_commit(smem_u32(&sh->s_full[b]));
          if (ct + 1 == hi) umma_commit(smem_u32(&sh->a_empty));
        }
      }
      umma_commit(smem_u32(&sh->drain));
      drain_wait(smem_u32(&sh->drain), 0, a.status);
    }
  } else {
    // ---------------- epilogue: warpgroup x owns row tile x ----------------
    const int x = (warp - 2) >> 2;
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int lrow = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    constexpr int BPT = 128 / CPB;          // KV blocks per column tile
    uint32_t t = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int e = item % kScore2Parts, bh = (item / kScore2Parts) / pairs, p = item / kScore2Parts - bh * pairs;
      const bool mine = x < n_rt(p);
      const int nct = tiles_for(p);
      int lo, hi;
      range_of(p, e, lo, hi);
      const int r = (2 * p + x) * 128 + lrow;
      const int pos = r * a.step;
      const int climit = a.causal ? min(a.cols, pos + 1) : a.cols;
      // this part's running LSE: row-LSE partial e (the select kernel
      // combines the partials in fp64)
      float M = -CUDART_INF_F, Ssum = 0.f;
      float* bl = a.blocklse + static_cast<int64_t>(bh) * a.nkb * a.rows + r;
      for (int ct = lo; ct < hi; ++ct, ++t) {
        const int b = t & 1;
        if (!warp_wait(smem_u32(&sh->s_full[b]), (t >> 1) & 1, abort, a.status, 44, item, ct, t, x)) { ok = false; break; }
        tc_fence_after();
        if (!mine) {
          tc_fence_before();
          mbar_arrive(smem_u32(&sh->s_empty[b]));
          continue;
        }
        uint32_t raw[128];
        tmem_ld128(tmem + x * 256 + b * 128 + lane_off, raw);
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->s_empty[b]));
        float* z = reinterpret_cast<float*>(raw);
        const int c0 = ct * 128;
        float blse[BPT];
        if (c0 + 128 <= climit) {
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) blse[bb] = block_lse<CPB, false>(z + bb * CPB, a.scale_log2);
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) z[c] = c0 + c < climit ? z[c] : -CUDART_INF_F;
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) blse[bb] = block_lse<CPB, true>(z + bb * CPB, a.scale_log2);
        }
        float mt = blse[0];
#pragma unroll
        for (int bb = 1; bb < BPT; ++bb) mt = fmaxf(mt, blse[bb]);
        if (mt != -CUDART_INF_F) {
          const float Mn = fmaxf(M, mt);
          float add = 0.f;
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) add += fast_exp2(blse[bb] - Mn);
          Ssum = Ssum * fast_exp2(M - Mn) + add;
          M = Mn;
        }
        if (r < a.rows) {
#pragma unroll
          for (int bb = 0; bb < BPT; ++bb) {
            const int J = ct * BPT + bb;
            if (J < a.nkb) bl[static_cast<int64_t>(J) * a.rows] = blse[bb];
          }
        }
      }
      if (!ok) break;
      if (mine && r < a.rows) {
        // column tiles never visited (causal) hold no probability
        if (e == kScore2Parts - 1)
          for (int J = nct * BPT; J < a.nkb; ++J) bl[static_cast<int64_t>(J) * a.rows] = -CUDART_INF_F;
        a.rowlse[(static_cast<int64_t>(e) * a.BHq + bh) * a.rows + r] =
            M == -CUDART_INF_F ? -CUDART_INF_F : M + __log2f(Ssum);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// a score row's log2-domain LSE from its n_part partials, in fp64
__device__ __forceinline__ double combine_partials(const SelectArgs& a, int bh, int r) {
  const int64_t plane = static_cast<int64_t>(a.B) * a.Hq * a.rows;
  const float* p = a.rowlse + static_cast<int64_t>(bh) * a.rows + r;
  double mx = -CUDART_INF;
  for (int e = 0; e < a.n_part; ++e) mx = fmax(mx, static_cast<double>(p[e * plane]));
  if (mx == -CUDART_INF) return mx;
  double sum = 0.0;
  for (int e = 0; e < a.n_part; ++e) sum += exp2(static_cast<double>(p[e * plane]) - mx);
  return mx + log2(sum);
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
  // row LSE: the two epilogue warpgroups of the score kernel each wrote the
  // LSE of the column tiles they handled; combine them (log2 domain)
  __shared__ double rlse[128];
  for (int s = threadIdx.x; s < nvalid; s += blockDim.x) {
    rlse[s] = combine_partials(a, bh, rbeg + s);
  }
  __syncthreads();

  for (int J = threadIdx.x; J < P2; J += blockDim.x) {
    if (J < a.nkb) {
      const float* bl = a.blocklse + (static_cast<int64_t>(bh) * a.nkb + J) * a.rows + rbeg;
      double m = 0.0;
      for (int s = 0; s < nvalid; ++s) {
        const float x = bl[s];
        if (x != -CUDART_INF_F) m += exp2_split(static_cast<double>(x) - rlse[s]);
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
  // rank policy: the visible blocks are the first n_vis ranks (blocks past
  // the diagonal have mass exactly 0 and lose ties to lower indices)
  const int n_vis = a.causal ? min(I + 1, a.nkb) : a.nkb;
  for (int i = k0; i < min(k0 + per, a.nkb); ++i) {
    const int J = static_cast<int>(key[i] & 0xFFFFFFFFu);
    const double mJ = scan[J];
    const double x = a.policy == 1 ? static_cast<double>(i) / static_cast<double>(n_vis) : C;
    int lev = 0;
    for (int l = 0; l < a.levels; ++l) lev += (static_cast<double>(a.thresholds[l]) <= x);
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

// ----------------------------------------------------------------------------
// select by buckets, one warp per (b, h, query block), up to 1024 key blocks.
// A block's level depends only on which thresholds its exclusive prefix C_J
// (or its rank) passes, so no full sort is needed:
// - the masses go into 256 buckets by their fraction of the row's largest
//   mass (larger mass, lower bucket, so the buckets keep the rank order);
//   exact zeros go into a bucket of their own after all others;
// - a histogram of counts and of 64-bit fixed-point mass sums, and its
//   exclusive scan, give every bucket's first prefix and first rank;
// - a bucket with no threshold inside the range of prefixes (or ranks) its
//   blocks can take gives them all one level;
// - the blocks of the few buckets a threshold falls into are listed,
//   grouped by bucket, and each counts the members of its own group that
//   rank before it to get its exact prefix and rank.
// Fixed-point sums are exact for masses above 2^-39 and do not depend on
// the order of the additions.  Everything per block lives in shared memory
// (no per-block registers), so every phase is a plain loop over the blocks.
// ----------------------------------------------------------------------------
constexpr int kBuckets = 256;                   // plus bucket 256 for exact zeros
constexpr int kBucketSlots = kBuckets + 2;      // slot 257 receives the totals
constexpr int kBucketWarps = 4;                 // rows (warps) per CTA
constexpr double kFix = 4611686018427387904.0;  // 2^62: fixed-point scale of a mass in [0, 1]

__device__ __forceinline__ unsigned long long mass_fix(float m) {
  return static_cast<unsigned long long>(static_cast<double>(m) * kFix);
}
// rank order: descending mass, then ascending index (masses are >= 0, so
// their bits order like the values)
__device__ __forceinline__ unsigned long long rank_key(float m, int J) {
  return (static_cast<unsigned long long>(0xFFFFFFFFu - __float_as_uint(m)) << 32) | static_cast<unsigned>(J);
}

// 2^x as exp2_split, with 2^n written into the exponent field directly
__device__ __forceinline__ double exp2_split_exp(double x) {
  if (x < -1000.0) return 0.0;
  const double n = floor(x);
  float p;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p) : "f"(static_cast<float>(x - n)));
  return static_cast<double>(p) * __longlong_as_double(static_cast<long long>(static_cast<int>(n) + 1023) << 52);
}

// per-warp shared memory of select_bucket_kernel (byte offsets), for
// P = nkb rounded up to 32 and R = score rows per query block (<= 128)
struct BucketLayout {
  int hs, tfx, rlse, mass, hc, lend, rth, list, ex, mixed, lv, bytes;
};
__host__ __device__ inline BucketLayout bucket_layout(int P, int R) {
  BucketLayout L{};
  int o = 0;
  L.hs = o;    o += 8 * kBucketSlots;   // u64 fixed-point sums, then their exclusive prefix
  L.tfx = o;   o += 8 * 8;              // u64 thresholds in fixed point
  L.rlse = o;  o += 8 * ((R + 1) & ~1); // f64 row LSEs of the row block's score rows
  L.mass = o;  o += 4 * P;              // f32 block masses
  L.hc = o;    o += 4 * kBucketSlots;   // counts, then the exclusive rank
  L.lend = o;  o += 4 * kBucketSlots;   // start of a bucket's list group, then its end
  L.rth = o;   o += 4 * 8;              // quantile policy: first rank of each level
  L.list = o;  o += 2 * P;              // u16 blocks of mixed buckets, grouped by bucket
  L.ex = o;    o += P;                  // exact level of every listed block
  L.mixed = o; o += kBucketSlots;       // a threshold falls inside the bucket
  L.lv = o;    o += kBucketSlots;       // the level of every block of an unmixed bucket
  L.bytes = (o + 15) & ~15;
  return L;
}

__global__ void __launch_bounds__(32 * kBucketWarps) select_bucket_kernel(const SelectArgs a) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int row = blockIdx.x * kBucketWarps + wid;              // (b*Hq + h)*nqb + I
  if (row >= a.B * a.Hq * a.nqb) return;
  const BucketLayout L = bucket_layout((a.nkb + 31) & ~31, a.rows_per_block);
  uint8_t* base = sel_smem + wid * L.bytes;
  unsigned long long* hs = reinterpret_cast<unsigned long long*>(base + L.hs);
  unsigned long long* tfx = reinterpret_cast<unsigned long long*>(base + L.tfx);
  double* rlse = reinterpret_cast<double*>(base + L.rlse);
  float* mass = reinterpret_cast<float*>(base + L.mass);
  int* hc = reinterpret_cast<int*>(base + L.hc);
  int* lend = reinterpret_cast<int*>(base + L.lend);
  int* rth = reinterpret_cast<int*>(base + L.rth);
  uint16_t* list = reinterpret_cast<uint16_t*>(base + L.list);
  uint8_t* ex = base + L.ex;
  uint8_t* mixed = base + L.mixed;
  uint8_t* lv = base + L.lv;

  const int bh = row / a.nqb, I = row - bh * a.nqb;
  const int b = bh / a.Hq, h = bh - b * a.Hq;
  const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int rbeg = I * a.rows_per_block;
  int nvalid;
  if (a.mode == 0) {
    nvalid = 0;
    for (int s = 0; s < a.rows_per_block; ++s) nvalid += (static_cast<int64_t>(rbeg + s) * a.step < a.N);
  } else {
    nvalid = min(a.rows_per_block, a.rows - rbeg);
  }
  for (int s = lane; s < nvalid; s += 32) {
    rlse[s] = combine_partials(a, bh, rbeg + s);
  }
  for (int i = lane; i < kBucketSlots; i += 32) {
    hs[i] = 0ull;
    hc[i] = 0;
  }
  if (lane < 8) {
    const float t = a.thresholds[lane];
    tfx[lane] = t >= 2.0f ? ~0ull : (t <= 0.0f ? 0ull : mass_fix(t));
  }
  __syncwarp();

  // block masses (the same arithmetic as select_kernel); with eight score
  // rows the next block's rows are loaded while this one is summed
  float mmax = 0.f;
  {
    const float* rowbase = a.blocklse + static_cast<int64_t>(bh) * a.nkb * a.rows + rbeg;
    const bool eight = nvalid == 8;
    float nx[8];
    if (eight && lane < a.nkb) {
#pragma unroll
      for (int u = 0; u < 8; ++u) nx[u] = __ldg(rowbase + static_cast<int64_t>(lane) * a.rows + u);
    }
    for (int J = lane; J < a.nkb; J += 32) {
      const float* bl = rowbase + static_cast<int64_t>(J) * a.rows;
      double m = 0.0;
      if (eight) {
        float cur[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[u] = nx[u];
        if (J + 32 < a.nkb) {
#pragma unroll
          for (int u = 0; u < 8; ++u) nx[u] = __ldg(bl + static_cast<int64_t>(32) * a.rows + u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (cur[u] != -CUDART_INF_F) m += exp2_split_exp(static_cast<double>(cur[u]) - rlse[u]);
      } else {
        // other row counts: groups of eight loads issued together, in row order
        int s = 0;
        for (; s + 8 <= nvalid; s += 8) {
          float x[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) x[u] = __ldg(bl + s + u);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (x[u] != -CUDART_INF_F) m += exp2_split_exp(static_cast<double>(x[u]) - rlse[s + u]);
        }
        for (; s < nvalid; ++s) {
          const float x = __ldg(bl + s);
          if (x != -CUDART_INF_F) m += exp2_split_exp(static_cast<double>(x) - rlse[s]);
        }
      }
      const float ms = static_cast<float>(m / nvalid);
      if (a.mass_out) a.mass_out[static_cast<int64_t>(row) * a.nkb + J] = ms;
      mass[J] = ms;
      mmax = fmaxf(mmax, ms);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  __syncwarp();
  // bucket of a block: any function monotone in the mass keeps the rank
  // order; the product by one reciprocal and the floor are (fp32 rounding is
  // monotone), and recomputing it gives the same bucket every time
  const float inv_max = mmax > 0.f ? 1.0f / mmax : 0.f;
  auto bucket_of = [&](float m) {
    return m == 0.f ? kBuckets
                    : max(0, min(kBuckets - 1, static_cast<int>(floorf(static_cast<float>(kBuckets) * (1.0f - m * inv_max)))));
  };

  // buckets (monotone in the mass: the fp32 quotient and product round
  // monotonically) and the histogram.  Exact zeros (every block past the
  // diagonal of a causal row) add nothing to the sums and are counted by a
  // ballot, not by atomics that would all hit one address.
  for (int j0 = 0; j0 < a.nkb; j0 += 32) {
    const int J = j0 + lane;
    const bool valid = J < a.nkb;
    const float m = valid ? mass[J] : 1.f;
    const unsigned zeros = __ballot_sync(0xffffffffu, m == 0.f);
    if (lane == 0 && zeros) atomicAdd(&hc[kBuckets], __popc(zeros));
    if (valid && m != 0.f) {
      const int bb = bucket_of(m);
      atomicAdd(&hc[bb], 1);
      atomicAdd(&hs[bb], mass_fix(m));
    }
  }
  __syncwarp();

  // exclusive scan over buckets 0..kBuckets; lane l owns buckets 9l .. 9l+8
  constexpr int PER = 9;                          // 32 * 9 = 288 >= kBuckets + 1
  {
    unsigned long long ls = 0ull;
    int lc = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int bb = lane * PER + i;
      if (bb <= kBuckets) { ls += hs[bb]; lc += hc[bb]; }
    }
    unsigned long long is = ls;
    int ic = lc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long ys = __shfl_up_sync(0xffffffffu, is, o);
      const int yc = __shfl_up_sync(0xffffffffu, ic, o);
      if (lane >= o) { is += ys; ic += yc; }
    }
    unsigned long long cs = is - ls;
    int cc = ic - lc;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int bb = lane * PER + i;
      if (bb <= kBuckets) {
        const unsigned long long vs = hs[bb];
        const int vc = hc[bb];
        hs[bb] = cs;
        hc[bb] = cc;
        cs += vs;
        cc += vc;
      }
    }
    if (lane == 31) { hs[kBuckets + 1] = is; hc[kBuckets + 1] = ic; }
  }
  __syncwarp();

  const int n_vis = a.causal ? min(I + 1, a.nkb) : a.nkb;
  // quantile policy: level l applies from rank r on when t_l <= r / n_vis
  // (an fp64 quotient, as the definition is written); the quotient never
  // decreases with r, so that set of ranks is [rth[l], inf) and every test
  // is one integer comparison.  ceil(t n) is within one of the boundary.
  if (a.policy == 1 && lane < a.levels) {
    const double t = static_cast<double>(a.thresholds[lane]);
    const double n = static_cast<double>(n_vis);
    int r;
    if (t <= 0.0) {
      r = 0;
    } else if (!(t < 2.0)) {
      r = 0x7FFFFFFF;                              // beyond every rank (r < n_vis <= 1024); NaN too
    } else {
      r = static_cast<int>(ceil(t * n));
      for (int it = 0; it < 4 && r > 0 && t <= static_cast<double>(r - 1) / n; ++it) --r;
      for (int it = 0; it < 4 && !(t <= static_cast<double>(r) / n); ++it) ++r;
    }
    rth[lane] = r;
  }
  __syncwarp();
  auto lev_rank = [&](int r) {
    int lev = 0;
    for (int l = 0; l < a.levels; ++l) lev += r >= rth[l];
    return lev;
  };
  auto lev_fix = [&](unsigned long long C) {
    int lev = 0;
    for (int l = 0; l < a.levels; ++l) lev += tfx[l] <= C;
    return lev;
  };

  // per bucket: mixed or not, the level of an unmixed one, and the start of
  // its list group (an exclusive scan of the mixed buckets' counts)
  int nmix;
  {
    int lsum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int bb = lane * PER + i;
      if (bb <= kBuckets) {
        const int c = hc[bb + 1] - hc[bb];
        bool mx = false;
        if (c > 0) {
          if (a.policy == 1) {
            mx = lev_rank(hc[bb]) != lev_rank(hc[bb + 1] - 1);
          } else if (bb < kBuckets) {             // exact zeros leave the prefix unchanged
            for (int l = 0; l < a.levels; ++l) mx |= (hs[bb] < tfx[l] && tfx[l] <= hs[bb + 1]);
          }
        }
        mixed[bb] = mx;
        lv[bb] = static_cast<uint8_t>(a.policy == 1 ? lev_rank(hc[bb]) : lev_fix(hs[bb]));
        lsum += mx ? c : 0;
      }
    }
    int incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    nmix = __shfl_sync(0xffffffffu, incl, 31);
    int off = incl - lsum;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int bb = lane * PER + i;
      if (bb <= kBuckets) {
        lend[bb] = off;
        off += mixed[bb] ? hc[bb + 1] - hc[bb] : 0;
      }
    }
  }
  __syncwarp();

  // list the blocks of mixed buckets (within a group in any order)
  if (nmix > 0) {
    for (int J = lane; J < a.nkb; J += 32) {
      const int bb = bucket_of(mass[J]);
      if (mixed[bb]) list[atomicAdd(&lend[bb], 1)] = static_cast<uint16_t>(J);
    }
    __syncwarp();
    // exact prefix / rank of every listed block from the members of its
    // group with a smaller rank key
    for (int i = lane; i < nmix; i += 32) {
      const int Jj = list[i];
      const unsigned long long kj = rank_key(mass[Jj], Jj);
      const int bj = bucket_of(mass[Jj]);
      const int end = lend[bj], beg = end - (hc[bj + 1] - hc[bj]);
      unsigned long long psum = 0ull;
      int pcnt = 0;
      for (int j = beg; j < end; ++j) {
        const int Jk = list[j];
        const float mk = mass[Jk];
        if (rank_key(mk, Jk) < kj) {
          psum += mass_fix(mk);
          ++pcnt;
        }
      }
      ex[Jj] = static_cast<uint8_t>(a.policy == 1 ? lev_rank(hc[bj] + pcnt) : lev_fix(hs[bj] + psum));
    }
    __syncwarp();
  }

  // levels, forced rules, the mask
  for (int J = lane; J < a.nkb; J += 32) {
    const int bb = bucket_of(mass[J]);
    const int lev = mixed[bb] ? ex[J] : lv[bb];
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
  }
}

}  // namespace

cudaError_t launch_score(const CUtensorMap* mapA, const CUtensorMap* mapB, const ScoreArgs& a, int num_sms,
                         cudaStream_t s) {
  const int row_tiles = (a.rows + 127) / 128;
  if (a.mode == 0 && a.d == 128) {
    // sampling: two row tiles per item share each K tile
    const int n2 = a.BHq * ((row_tiles + 1) / 2) * kScore2Parts;
    const int grid2 = n2 < num_sms ? n2 : num_sms;
    const size_t smem2 = 1024 + kRegion2 * kChunk + sizeof(Score2Shared);
    switch (a.cols_per_block) {
#define PSA_SCORE2_CASE(CPB)                                                                       \
  case CPB: {                                                                                      \
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(score2_kernel<CPB>),            \
                                   static_cast<int>(smem2));                                       \
    if (e != cudaSuccess) return e;                                                                \
    score2_kernel<CPB><<<grid2, kThreads, smem2, s>>>(*mapA, *mapB, a);                            \
    return cudaGetLastError();                                                                     \
  }
      PSA_SCORE2_CASE(64)
      PSA_SCORE2_CASE(128)
#undef PSA_SCORE2_CASE
      default: break;
    }
  }
  const int n_items = a.BHq * row_tiles;
  const int grid = n_items < num_sms ? n_items : num_sms;
  const size_t smem = 1024 + kRegionChunks * kChunk + sizeof(ScoreShared);
  switch (a.cols_per_block) {
#define PSA_SCORE_CASE(CPB)                                                                       \
  case CPB: {                                                                                     \
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(score_kernel<CPB>),             \
                                   static_cast<int>(smem));                                       \
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
  // rows_per_block <= 128 always (8 sampled rows, 1 mean row, or block / S
  // antidiagonal groups), which both kernels' row-LSE arrays rely on
  if (a.rows_per_block > 128) return cudaErrorInvalidValue;
  if (a.nkb <= 1024) {
    const size_t smem = static_cast<size_t>(kBucketWarps) * bucket_layout((a.nkb + 31) & ~31, a.rows_per_block).bytes;
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(&select_bucket_kernel), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    select_bucket_kernel<<<(rows + kBucketWarps - 1) / kBucketWarps, 32 * kBucketWarps, smem, s>>>(a);
  } else {
    select_kernel<<<rows, kSelThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace psa
