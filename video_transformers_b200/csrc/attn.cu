// attn.cu -- stage 3 of the PSA forward path: adaptive pyramid attention
// (summary article "PSA: Pyramid Sparse Attention ...", Method: every KV
// block is read at the pyramid level the mask assigns it and a scale factor
// keeps the probabilities consistent; the kernel separates the logical block
// size from the hardware tile size; news review, Methodology 4: ordinary
// scaled dot-product attention over the pooled KV).
//
// Two persistent CTAs per SM, 6 warps each.  A work item is a 128-row query
// tile; its KV side is the planner's list of 128-row KV tiles, processed as
// 64-row sub-tiles so that one sub-tile's S = Q K^T runs on the tensor core
// while the softmax works on the previous one.
//   warp 0      TMA producer.  Per sub-tile: one box per (segment, 64-channel
//               chunk) of the level-l K and V maps, issued by the lane that
//               owns the segment, into two-stage K and V rings; plus a small
//               record of the sub-tile (the level of each 16-column chunk, or
//               a per-column bias/validity when it holds padding, a ragged
//               block, a causal edge or a query-half mask).
//   warp 1      tcgen05 issuer (one thread): S_j = Q K_j^T (M 128, N 64) into
//               one of two TMEM S buffers, then O += P_{j-1} V_{j-1} with P
//               read from TMEM.
//   warps 2..5  softmax, one query row per thread: exp2 argument
//               s * scale * log2(e) + l - m (the +ln 2^l bias in log2 units),
//               lazy rescaling of O in TMEM, P as bf16 back into the S buffer,
//               and the final O / l and lse store.
// TMEM per CTA: S buffers at columns [0, 64) and [64, 128), O at [128, 128+D).
// Every wait is bounded; a time-out sets the workspace status word and
// records where it happened.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "attn_common.cuh"
#include "exp2_poly.h"
#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kThreads = 192;
constexpr int kSub = 64;                    // KV rows per sub-tile
constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 2^(8+3)
// With e4m3 probabilities the reference max moves in whole binades and at
// most 5 below the running max, so P <= 2^(5+3) stays under e4m3's 448.
constexpr float kRescaleThresholdP8 = 5.0f;
// Of every 8 column pairs of a full sub-tile, this many take their
// exponential on the FMA pipe (exp2_fma2) instead of the special-function
// unit.  Measured on B200 the special-function unit is not the limit of
// this kernel, so the default is none.
#ifndef PSA_POLY_PAIRS
#define PSA_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = PSA_POLY_PAIRS;

struct AttnMaps {
  CUtensorMap m[9];
};

// NST: depth of the K, V and sub-tile-record rings
template <int NST>
struct AttnShared {
  uint64_t q_full, q_empty;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t i_full[NST], i_empty[NST];
  uint64_t s_full[2], p_full[2];
  uint64_t o_ready, o_final, o_free, drain;
  uint64_t never;       // no thread ever arrives here (the debug trap of the time-out path)
  uint32_t tmem_base;
  int abort;
  SubInfo ti[NST];
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for two lanes at once on the FMA pipe, x <= 20: Cody-Waite split
// x = n + f with n = round(x) (adding 1.5 * 2^23 rounds to an integer in the
// low mantissa bits) and f in [-1/2, 1/2]; 2^f from the Remez polynomial of
// exp2_poly.h; 2^n added to the exponent field as an integer.  Inputs below
// -126 are clamped there (the result is then <= 2^-126, not 0), so it is
// used only where every column is a real key.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
  const float2 n = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(kExp2Poly3, kExp2Poly3), f, make_float2(kExp2Poly2, kExp2Poly2));
  p = __ffma2_rn(p, f, make_float2(kExp2Poly1, kExp2Poly1));
  p = __ffma2_rn(p, f, make_float2(kExp2Poly0, kExp2Poly0));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// P for one sub-tile row: p = 2^(s * sc + cb[k] - mu) per 16-column chunk k,
// packed to bf16 pairs; returns the row sum of p (fp32).
template <int POLY>
__device__ __forceinline__ float sub_probs(const float* s, float sc, const float (&cb)[4], float mu,
                                           uint32_t (&pk)[32]) {
  const float2 sc2 = make_float2(sc, sc);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 off = make_float2(cb[k] - mu, cb[k] - mu);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 x = __ffma2_rn(make_float2(s[16 * k + 2 * i], s[16 * k + 2 * i + 1]), sc2, off);
      float2 p;
      if (i < POLY) {
        p = exp2_fma2(x);
      } else {
        p.x = fast_exp2(x.x);
        p.y = fast_exp2(x.y);
      }
      acc[i & 3] = __fadd2_rn(acc[i & 3], p);
      pk[8 * k + i] = pack_bf16(p.x, p.y);
    }
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

// two fp32 values as e4m3 codes (nearest, ties to even, saturating): lo in
// the low byte, hi in the high byte
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// sub_probs with the probabilities rounded to e4m3, four per 32-bit word
// (column c in byte c % 4 of word c / 4: the 8-bit A-operand layout of a TS
// MMA); returns the sum of the unrounded fp32 probabilities
__device__ __forceinline__ float sub_probs8(const float* s, float sc, const float (&cb)[4], float mu,
                                            uint32_t (&pk)[16]) {
  const float2 sc2 = make_float2(sc, sc);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 off = make_float2(cb[k] - mu, cb[k] - mu);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float2 x0 = __ffma2_rn(make_float2(s[16 * k + 2 * i], s[16 * k + 2 * i + 1]), sc2, off);
      const float2 x1 = __ffma2_rn(make_float2(s[16 * k + 2 * i + 2], s[16 * k + 2 * i + 3]), sc2, off);
      const float2 p0 = make_float2(fast_exp2(x0.x), fast_exp2(x0.y));
      const float2 p1 = make_float2(fast_exp2(x1.x), fast_exp2(x1.y));
      acc[i & 3] = __fadd2_rn(acc[i & 3], p0);
      acc[(i + 1) & 3] = __fadd2_rn(acc[(i + 1) & 3], p1);
      pk[4 * k + i / 2] = e4m3x2(p0.x, p0.y) | (e4m3x2(p1.x, p1.y) << 16);
    }
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

// 2^x for a whole number x <= 0, exactly (0 below the normal range)
__device__ __forceinline__ float exp2_whole(float x) {
  return x < -126.0f ? 0.0f : __int_as_float((127 + static_cast<int>(x)) << 23);
}

// number of 64-row sub-tiles of an item with `rows` real KV rows
__device__ __forceinline__ uint32_t sub_count(int rows) { return static_cast<uint32_t>((rows + kSub - 1) / kSub); }

// H2: the query tile holds two 64-token query blocks whose segment lists
// differ, so records are kept per query half (block 64); with 128-token
// blocks both halves always agree and the per-half work is compiled out.
// QK8: the FP8 path.  Q and K arrive as e4m3 codes (128-byte rows at d = 128,
// one 128-byte-swizzled chunk), S = Q K^T runs as kind::f8f6f4 MMAs (K = 32
// per instruction), and the softmax scale of a row carries the row's query
// scale times its KV head's key scale; V, P and O are as in the bf16 path.
// PV8 (with QK8): V arrives as e4m3 codes too (one 128-byte-swizzled chunk
// per 64-row stage) and O += P V runs as kind::f8f6f4 MMAs (K = 32) with P
// as e4m3 in TMEM and V as an MN-major B operand; the reference max moves
// in whole binades (P's e4m3 rounding then does not depend on when it
// moved), and the output carries the KV head's value scale.
template <int D, bool OUT_F32, int NST, int CTAS, bool H2, bool QK8 = false, bool PV8 = false>
__global__ void __launch_bounds__(kThreads, CTAS)
    attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  static_assert(!QK8 || D == 128, "the FP8 path is built for d = 128");
  static_assert(!PV8 || QK8, "e4m3 probabilities come with e4m3 queries and keys");
  constexpr int QB = QK8 ? D * 128 : D * 256;    // bytes of the 128-row Q tile
  constexpr int SBK = QK8 ? D * 64 : D * 128;    // bytes of a 64-row K stage
  constexpr int SB = PV8 ? D * 64 : D * 128;     // bytes of a 64-row V stage
  constexpr int KC = D / 64;                     // 64-channel bf16 chunks
  constexpr uint32_t kTmemCols = 256;
  using Shared = AttnShared<NST>;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + QB;               // NST stages
  uint8_t* sV = sK + NST * SBK;        // NST stages
  Shared* sh = reinterpret_cast<Shared*>(sV + NST * SB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = a.levels;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->q_full), 1);
    mbar_init(smem_u32(&sh->q_empty), 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(smem_u32(&sh->k_full[i]), 1);
      mbar_init(smem_u32(&sh->k_empty[i]), 1);
      mbar_init(smem_u32(&sh->v_full[i]), 1);
      mbar_init(smem_u32(&sh->v_empty[i]), 1);
      mbar_init(smem_u32(&sh->i_full[i]), 32);
      mbar_init(smem_u32(&sh->i_empty[i]), 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh->s_full[i]), 1);
      mbar_init(smem_u32(&sh->p_full[i]), 128);
    }
    mbar_init(smem_u32(&sh->o_ready), 1);
    mbar_init(smem_u32(&sh->o_final), 1);
    mbar_init(smem_u32(&sh->o_free), 128);
    mbar_init(smem_u32(&sh->drain), 1);
    mbar_init(smem_u32(&sh->never), 1);
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&sh->tmem_base), kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t tO = tmem + 128;
  volatile int* abort = &sh->abort;

  if (warp == 0) {
    // =============================== producer ===============================
    if (lane == 0) {
      for (int i = 0; i < 1 + 2 * L; ++i) tma_prefetch_desc(&maps.m[i]);
    }
    uint32_t it = 0, qcnt = 0;       // it: sub-tiles loaded so far
    uint32_t kiss = 0, viss = 0;     // K and V sub-tile loads issued (the drain waits for exactly these)
    bool trap = debug_wait_trap(a.status);
    bool ok = true;
    for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
      const int item = a.queue[idx];
      const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
      if (t1 == t0) continue;
      const uint32_t nsub = sub_count(a.item_rows[item]);
      const int bh = item / a.n_qtiles, tq = item - bh * a.n_qtiles;
      const int b = bh / a.Hq, h = bh - b * a.Hq;
      const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
      const int q0 = tq * 128;
      if (!warp_wait(smem_u32(&sh->q_empty), (qcnt & 1) ^ 1, abort, a.status, 11, idx, qcnt, it, 0)) { ok = false; break; }
      if (lane == 0) {
        const uint32_t bar = smem_u32(&sh->q_full);
        mbar_arrive_expect_tx(bar, QB);
        if (QK8) {
          tma_load_3d(smem_u32(sQ), &maps.m[0], bar, 0, q0, bh);
        } else {
#pragma unroll
          for (int kc = 0; kc < KC; ++kc) tma_load_3d(smem_u32(sQ + kc * 16384), &maps.m[0], bar, kc * 64, q0, bh);
        }
      }
      ++qcnt;
      // V loads run one sub-tile behind the K loads: V_j is needed only after
      // the softmax of sub-tile j, while K_{j+1} is needed right after S_j.
      bool pv_mine = false;
      int pv_l = 0, pv_dst = 0, pv_prow = 0;
      // segment words of the current tile, and of the next one (prefetched)
      int sb = a.tile_seg_off[t0], nseg = a.tile_seg_off[t0 + 1] - sb;
      int w = lane < nseg ? a.segs[sb + lane] : 0;
      int nb = 0, nn = 0, wn = 0;
      int l = 0, half = 0, J = 0, rows = 0, r = 0;
      for (uint32_t j = 0; j < nsub && ok; ++j, ++it) {
        const int t = t0 + static_cast<int>(j >> 1);
        const int hs = static_cast<int>(j & 1);          // which 64-row half of the KV tile
        if (hs == 0) {
          if (j > 0) { sb = nb; nseg = nn; w = wn; }
          // this tile's segments: lane s owns segment s (at most 16)
          l = seg_level(w); half = seg_half(w); J = seg_block(w);
          rows = lane < nseg ? (a.block >> l) : 0;
          r = rows;                                     // inclusive scan -> exclusive row offset
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, r, o);
            if (lane >= o) r += y;
          }
          r -= rows;
          if (t + 1 < t1) { nb = a.tile_seg_off[t + 1]; nn = a.tile_seg_off[t + 2] - nb; }
        } else if (t + 1 < t1) {
          wn = lane < nn ? a.segs[nb + lane] : 0;
        }
        const int nl = a.N >> l;
        // part of the segment inside this half: rows [lo, lo + cnt) of the segment at sub-tile row dst
        bool mine;
        int lo, dst, cnt;
        if (rows > kSub) { mine = lane < nseg; lo = hs * kSub; dst = 0; cnt = kSub; }
        else { mine = lane < nseg && (r >> 6) == hs; lo = 0; dst = r - hs * kSub; cnt = rows; }
        const int prow = (half ? J * rows : nl) + lo;   // padding reads past the end: zeros
        const int st = it % NST;
        const uint32_t ph = (it / NST) & 1;

        // K
        if (!warp_wait(smem_u32(&sh->k_empty[st]), ph ^ 1, abort, a.status, 12, idx, j, it, 0)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(smem_u32(&sh->k_full[st]), SBK);
        __syncwarp();
        if (mine) {
          if (QK8) {
            tma_load_3d(smem_u32(sK + st * SBK + dst * 128), &maps.m[1 + l], smem_u32(&sh->k_full[st]), 0, prow, hkv);
          } else {
#pragma unroll
            for (int kc = 0; kc < KC; ++kc)
              tma_load_3d(smem_u32(sK + st * SBK + kc * 8192 + dst * 128), &maps.m[1 + l], smem_u32(&sh->k_full[st]),
                          kc * 64, prow, hkv);
          }
        }
        ++kiss;
        if (trap) {
          // debug trap: with a K load in flight, wait on a barrier no thread
          // arrives at, so that the wait runs out (after the debug limit,
          // long before any other wait could) and the CTA unwinds
          trap = false;
          if (!warp_wait(smem_u32(&sh->never), 0, abort, a.status, 10, idx, j, it, 0, debug_trap_limit(a.status))) {
            ok = false;
            break;
          }
        }

        // sub-tile record
        if (!warp_wait(smem_u32(&sh->i_empty[st]), ph ^ 1, abort, a.status, 13, idx, j, it, 0)) { ok = false; break; }
        SubInfo& ti = sh->ti[st];
        write_subinfo<H2>(ti, lane, mine, half, l, J, rows, lo, cnt, dst, w, nseg, nl, q0, a.N, a.block, a.causal);
        mbar_arrive(smem_u32(&sh->i_full[st]));

        // V of the previous sub-tile
        if (j > 0) {
          const uint32_t pst = (it - 1) % NST;
          if (!warp_wait(smem_u32(&sh->v_empty[pst]), (((it - 1) / NST) & 1) ^ 1, abort, a.status, 14, idx, j, it, 0)) { ok = false; break; }
          if (lane == 0) mbar_arrive_expect_tx(smem_u32(&sh->v_full[pst]), SB);
          __syncwarp();
          if (pv_mine) {
            if (PV8) {
              tma_load_3d(smem_u32(sV + pst * SB + pv_dst * 128), &maps.m[1 + L + pv_l], smem_u32(&sh->v_full[pst]), 0,
                          pv_prow, hkv);
            } else {
#pragma unroll
              for (int kc = 0; kc < KC; ++kc)
                tma_load_3d(smem_u32(sV + pst * SB + kc * 8192 + pv_dst * 128), &maps.m[1 + L + pv_l],
                            smem_u32(&sh->v_full[pst]), kc * 64, pv_prow, hkv);
            }
          }
          ++viss;
        }
        pv_mine = mine; pv_l = l; pv_dst = dst; pv_prow = prow;
      }
      // V of the item's last sub-tile
      if (ok) {
        const uint32_t pst = (it - 1) % NST;
        if (!warp_wait(smem_u32(&sh->v_empty[pst]), (((it - 1) / NST) & 1) ^ 1, abort, a.status, 15, idx, 0, it, 0)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(smem_u32(&sh->v_full[pst]), SB);
        __syncwarp();
        if (pv_mine) {
          if (PV8) {
            tma_load_3d(smem_u32(sV + pst * SB + pv_dst * 128), &maps.m[1 + L + pv_l], smem_u32(&sh->v_full[pst]), 0,
                        pv_prow, hkv);
          } else {
#pragma unroll
            for (int kc = 0; kc < KC; ++kc)
              tma_load_3d(smem_u32(sV + pst * SB + kc * 8192 + pv_dst * 128), &maps.m[1 + L + pv_l],
                          smem_u32(&sh->v_full[pst]), kc * 64, pv_prow, hkv);
          }
        }
        ++viss;
      }
    }
    // drain: every TMA this warp issued must land before the CTA exits.  The
    // k-th K (V) load went to stage k % NST, phase k / NST, so the last load
    // of stage st is number kiss - 1 - ((kiss - 1 - st) % NST) and its phase
    // parity is ((kiss - 1 - st) / NST) & 1.  K and V are counted apart: after
    // an abort the V ring trails the K ring by one load.
    if (lane == 0) {
      if (qcnt > 0) drain_wait(smem_u32(&sh->q_full), (qcnt - 1) & 1, a.status);
      for (uint32_t st = 0; st < static_cast<uint32_t>(NST); ++st) {
        if (kiss > st) drain_wait(smem_u32(&sh->k_full[st]), ((kiss - 1 - st) / NST) & 1, a.status);
        if (viss > st) drain_wait(smem_u32(&sh->v_full[st]), ((viss - 1 - st) / NST) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, kSub, false);
      constexpr uint32_t idS8 = idesc_e4m3_f32(128, kSub);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
      constexpr uint32_t idO8 = idesc_e4m3_f32(128, D, true);
      uint32_t it = 0, qcnt = 0, icnt = 0;
      bool ok = true;
      // shared-memory descriptors of the tile bases; a K step or stage is an
      // offset added to the start-address field (all of smem is < 256 KB)
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 8192, 1024);
      // O += P_jj V_jj for sub-tile jj of the current item
      auto issue_pv = [&](uint32_t jj, bool first_of_item) -> bool {
        const uint32_t g = it + jj, st = g % NST, sb2 = g & 1;
        if (first_of_item && icnt > 0) {
          if (!bounded_wait(smem_u32(&sh->o_free), (icnt - 1) & 1, abort, a.status, 21, icnt, jj, g, 0)) return false;
        }
        if (!bounded_wait(smem_u32(&sh->p_full[sb2]), (g >> 1) & 1, abort, a.status, 22, icnt, jj, g, 0)) return false;
        if (!bounded_wait(smem_u32(&sh->v_full[st]), (g / NST) & 1, abort, a.status, 26, icnt, jj, g, 0)) return false;
        tc_fence_after();
        if (PV8) {
          // K = 32 rows of V (4 KB of the stage) and 8 TMEM columns of P per MMA
#pragma unroll
          for (int k = 0; k < kSub / 32; ++k)
            umma_ts_f8(tO, tmem + sb2 * kSub + k * 8, dV + ((st * SB + k * 4096) >> 4), idO8,
                       (first_of_item && k == 0) ? 0u : 1u);
        } else {
#pragma unroll
          for (int k = 0; k < kSub / 16; ++k) {
            umma_ts(tO, tmem + sb2 * kSub + k * 8, dV + ((st * SB + k * 2048) >> 4), idO,
                    (first_of_item && k == 0) ? 0u : 1u);
          }
        }
        umma_commit(smem_u32(&sh->v_empty[st]));
        umma_commit(smem_u32(&sh->o_ready));
        return true;
      };
      for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
        const int item = a.queue[idx];
        const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
        if (t1 == t0) continue;
        const uint32_t n = sub_count(a.item_rows[item]);
        if (!bounded_wait(smem_u32(&sh->q_full), qcnt & 1, abort, a.status, 23, idx, qcnt, it, 0)) { ok = false; break; }
        tc_fence_after();
        ++qcnt;
        for (uint32_t j = 0; j < n && ok; ++j) {
          const uint32_t g = it + j, st = g % NST, sb2 = g & 1;
          // S_j = Q K_j^T into S buffer sb2
          if (!bounded_wait(smem_u32(&sh->k_full[st]), (g / NST) & 1, abort, a.status, 24, idx, j, g, 0)) { ok = false; break; }
          tc_fence_after();
          if (QK8) {
#pragma unroll
            for (int k = 0; k < D / 32; ++k)
              umma_ss_f8(tmem + sb2 * kSub, dQ + ((32 * k) >> 4), dK + ((st * SBK + 32 * k) >> 4), idS8, k != 0);
          } else {
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                umma_ss(tmem + sb2 * kSub, dQ + ((kc * 16384 + 32 * k) >> 4),
                        dK + ((st * SBK + kc * 8192 + 32 * k) >> 4), idS, (kc | k) != 0);
              }
            }
          }
          umma_commit(smem_u32(&sh->s_full[sb2]));
          umma_commit(smem_u32(&sh->k_empty[st]));
          if (j + 1 == n) umma_commit(smem_u32(&sh->q_empty));
          if (j >= 1 && !issue_pv(j - 1, j == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(n - 1, n == 1)) { ok = false; break; }
        umma_commit(smem_u32(&sh->o_final));
        it += n;
        ++icnt;
      }
      umma_commit(smem_u32(&sh->drain));
      drain_wait(smem_u32(&sh->drain), 0, a.status);
    }
  } else {
    // =============================== softmax ===============================
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int my_half = H2 ? (row >> 6) : 0;   // which query block of a 64-token-block tile
    uint32_t it = 0, icnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
      const int item = a.queue[idx];
      const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
      const int bh = item / a.n_qtiles, tq = item - bh * a.n_qtiles;
      const int tok = tq * 128 + row;
      const int64_t orow = static_cast<int64_t>(bh) * a.N + tok;
      if (t1 == t0) {
        if (tok < a.N) {
          if (OUT_F32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow * D);
            for (int c = 0; c < D / 4; ++c) o[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
            uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D);
            for (int c = 0; c < D / 8; ++c) o[c] = make_uint4(0u, 0u, 0u, 0u);
          }
          if (a.lse) a.lse[orow] = -CUDART_INF_F;
        }
        continue;
      }
      const uint32_t n = sub_count(a.item_rows[item]);
      float m = -CUDART_INF_F, lsum = 0.f;
      // softmax scale of this row (log2 units); the FP8 path folds in the
      // row's query scale and its KV head's key scale
      float row_sc = a.scale_log2;
      float out_sc = 1.0f;          // the KV head's value scale (e4m3 values only)
      if (QK8) {
        const int b = bh / a.Hq, h = bh - b * a.Hq;
        const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
        row_sc *= (tok < a.N ? a.qscale[orow] : 0.f) * a.kscale[hkv];
        if (PV8) out_sc = a.vscale[hkv];
      }
      for (uint32_t j = 0; j < n; ++j, ++it) {
        const uint32_t st = it % NST, sb2 = it & 1;
        if (!warp_wait(smem_u32(&sh->s_full[sb2]), (it >> 1) & 1, abort, a.status, 31, idx, j, it, 0)) { ok = false; break; }
        if (!warp_wait(smem_u32(&sh->i_full[st]), (it / NST) & 1, abort, a.status, 32, idx, j, it, 0)) { ok = false; break; }
        tc_fence_after();
        const SubInfo& ti = sh->ti[st];
        uint32_t sr[32], sr2[32];
        tmem_ld32(tmem + sb2 * kSub + lane_off, sr);
        tmem_ld32(tmem + sb2 * kSub + 32 + lane_off, sr2);
        float s[kSub];
#pragma unroll
        for (int i = 0; i < 32; ++i) { s[i] = __uint_as_float(sr[i]); s[32 + i] = __uint_as_float(sr2[i]); }
        // exp2 argument of column c in chunk k: s[c] * sc + cb[k] - m
        float sc = row_sc;
        float cb[4];
        float mt;
        const bool fast_tile = ti.fast != 0;
        if (fast_tile) {
          const float4 c4 = *reinterpret_cast<const float4*>(ti.cb[my_half]);
          cb[0] = c4.x; cb[1] = c4.y; cb[2] = c4.z; cb[3] = c4.w;
          float cmax[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float* x = s + 16 * k;
            const float y0 = fmax3(x[0], x[1], x[2]), y1 = fmax3(x[3], x[4], x[5]), y2 = fmax3(x[6], x[7], x[8]);
            const float y3 = fmax3(x[9], x[10], x[11]), y4 = fmax3(x[12], x[13], x[14]);
            cmax[k] = fmaf(fmax3(fmax3(y0, y1, y2), fmax3(y3, y4, x[15]), y0), sc, cb[k]);
          }
          mt = fmaxf(fmaxf(cmax[0], cmax[1]), fmaxf(cmax[2], cmax[3]));
        } else {
          // per-column bias (padding, ragged tails) and, if needed, the
          // causal / query-half test; afterwards s holds the full argument
#pragma unroll
          for (int c4 = 0; c4 < kSub / 4; ++c4) {
            const float4 bv = *reinterpret_cast<const float4*>(&ti.bias[my_half][4 * c4]);
            s[4 * c4 + 0] = fmaf(s[4 * c4 + 0], sc, bv.x);
            s[4 * c4 + 1] = fmaf(s[4 * c4 + 1], sc, bv.y);
            s[4 * c4 + 2] = fmaf(s[4 * c4 + 2], sc, bv.z);
            s[4 * c4 + 3] = fmaf(s[4 * c4 + 3], sc, bv.w);
          }
          if (ti.causal_check) {
#pragma unroll
            for (int c4 = 0; c4 < kSub / 4; ++c4) {
              const int4 iv = *reinterpret_cast<const int4*>(&ti.info[4 * c4]);
              s[4 * c4 + 0] = iv.x <= tok ? s[4 * c4 + 0] : -CUDART_INF_F;
              s[4 * c4 + 1] = iv.y <= tok ? s[4 * c4 + 1] : -CUDART_INF_F;
              s[4 * c4 + 2] = iv.z <= tok ? s[4 * c4 + 2] : -CUDART_INF_F;
              s[4 * c4 + 3] = iv.w <= tok ? s[4 * c4 + 3] : -CUDART_INF_F;
            }
          }
          sc = 1.0f;
#pragma unroll
          for (int k = 0; k < 4; ++k) cb[k] = 0.f;
          float x[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) x[u] = fmax3(s[u], s[8 + u], s[16 + u]);
#pragma unroll
          for (int c = 24; c < kSub; c += 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = fmax3(x[u], s[c + u], c + 8 + u < kSub ? s[c + 8 + u] : x[u]);
          }
          mt = fmaxf(fmax3(x[0], x[1], x[2]), fmax3(fmax3(x[3], x[4], x[5]), x[6], x[7]));
        }
        // the sub-tile record may be reused once read
        mbar_arrive(smem_u32(&sh->i_empty[st]));

        const float mnew = fmaxf(m, mt);
        // Lazy rescaling: a row moves its reference max only when the new max
        // exceeds it by more than kRescaleThreshold (or on its first visible
        // key).  O is read and written with warp-collective tcgen05.ld/st, so
        // the decision to touch O is taken per warp, after the PV of the
        // previous sub-tile is done (o_ready: PV_{j-2} completed before S_j,
        // PV_j waits for this sub-tile's P, so the awaited phase is one of
        // the two the barrier can be in).
        const bool first = m == -CUDART_INF_F && mnew != -CUDART_INF_F;
        const bool grow = m != -CUDART_INF_F && mnew > m + (PV8 ? kRescaleThresholdP8 : kRescaleThreshold);
        // e4m3 probabilities: the reference is the next whole binade
        const float mref = PV8 ? ceilf(mnew) : mnew;
        if (__any_sync(0xffffffffu, grow)) {
          const float f = grow ? (PV8 ? exp2_whole(m - mref) : fast_exp2(m - mnew)) : 1.0f;
          lsum *= f;
          if (grow) m = mref;
          if (!warp_wait(smem_u32(&sh->o_ready), (it - 1) & 1, abort, a.status, 33, idx, j, it, 0)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32 + lane_off, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tO + c * 32 + lane_off, o);
          }
        }
        if (first) m = mref;
        const float mu = m == -CUDART_INF_F ? 0.f : m;
        if (PV8) {
          uint32_t pk8[16];
          lsum += sub_probs8(s, sc, cb, mu, pk8);
          tmem_st16(tmem + sb2 * kSub + lane_off, pk8);
        } else {
          uint32_t pk[32];
          // sub-tiles with masked columns (p must be exactly 0 there) use the
          // special-function unit only
          lsum += fast_tile ? sub_probs<kPolyPairs>(s, sc, cb, mu, pk) : sub_probs<0>(s, sc, cb, mu, pk);
          tmem_st32(tmem + sb2 * kSub + lane_off, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->p_full[sb2]));
      }
      if (!ok) break;
      // epilogue: O / l once the item's last PV is done (o_final completes
      // once per item and cannot run ahead: the next item's first PV waits
      // for o_free)
      if (!warp_wait(smem_u32(&sh->o_final), icnt & 1, abort, a.status, 35, idx, n, it, icnt)) { ok = false; break; }
      ++icnt;
      tc_fence_after();
      const float inv = lsum > 0.f ? out_sc / lsum : 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32 + lane_off, o);
        if (tok < a.N) {
          if (OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow * D + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                   __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              v.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              v.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              v.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              dst[i] = v;
            }
          }
        }
      }
      if (a.lse && tok < a.N)
        a.lse[orow] = lsum > 0.f ? (m + __log2f(lsum)) * 0.69314718055994531f : -CUDART_INF_F;
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->o_free));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Resident CTAs per SM and ring depth.  Measured on B200 (Wan2.1-14B-shaped
// problem): two CTAs per SM with two-stage rings run 1.75x faster than one
// CTA per SM with five-stage rings; each CTA's S -> softmax -> PV chain has a
// fixed latency per sub-tile that only a second CTA hides.
#ifndef PSA_ATTN_CTAS
#define PSA_ATTN_CTAS 2
#endif

template <int D, bool F32, bool QK8 = false, bool PV8 = false>
cudaError_t launch_one(const AttnMaps& maps, const AttnArgs& a, int num_sms, cudaStream_t s) {
  constexpr int CTAS = PSA_ATTN_CTAS;
  constexpr int NST = CTAS == 1 ? (D == 128 ? 5 : 8) : 2;
  constexpr size_t QB = QK8 ? static_cast<size_t>(D) * 128 : static_cast<size_t>(D) * 256;
  constexpr size_t SBK = QK8 ? static_cast<size_t>(D) * 64 : static_cast<size_t>(D) * 128;
  constexpr size_t SBV = PV8 ? static_cast<size_t>(D) * 64 : static_cast<size_t>(D) * 128;
  const size_t smem = 1024 + QB + NST * (SBK + SBV) + sizeof(AttnShared<NST>);
  const int grid = a.n_items < CTAS * num_sms ? a.n_items : CTAS * num_sms;
  if (a.block == 64) {
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(attn_kernel<D, F32, NST, CTAS, true, QK8, PV8>),
                                   static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attn_kernel<D, F32, NST, CTAS, true, QK8, PV8><<<grid, kThreads, smem, s>>>(maps, a);
  } else {
    cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(attn_kernel<D, F32, NST, CTAS, false, QK8, PV8>),
                                   static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attn_kernel<D, F32, NST, CTAS, false, QK8, PV8><<<grid, kThreads, smem, s>>>(maps, a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap* maps, const AttnArgs& a, int num_sms, cudaStream_t s) {
  AttnMaps m;
  for (int i = 0; i < 1 + 2 * a.levels; ++i) m.m[i] = maps[i];
  for (int i = 1 + 2 * a.levels; i < 9; ++i) m.m[i] = maps[0];
  if (a.d == 128) return a.out_fp32 ? launch_one<128, true>(m, a, num_sms, s) : launch_one<128, false>(m, a, num_sms, s);
  return a.out_fp32 ? launch_one<64, true>(m, a, num_sms, s) : launch_one<64, false>(m, a, num_sms, s);
}

cudaError_t launch_attention_fp8(const CUtensorMap* maps, const AttnArgs& a, bool pv, int num_sms, cudaStream_t s) {
  if (a.d != 128 || a.out_fp32) return cudaErrorInvalidValue;
  AttnMaps m;
  for (int i = 0; i < 1 + 2 * a.levels; ++i) m.m[i] = maps[i];
  for (int i = 1 + 2 * a.levels; i < 9; ++i) m.m[i] = maps[0];
  return pv ? launch_one<128, false, true, true>(m, a, num_sms, s) : launch_one<128, false, true, false>(m, a, num_sms, s);
}

}  // namespace psa
