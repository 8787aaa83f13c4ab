// attn_dq.cu -- dQ of adaptive pyramid attention, query-major on the forward's
// tile plan (the derivative of the forward of the summary article "PSA:
// Pyramid Sparse Attention ...", Method, with the mask held fixed; news
// review, Methodology 4: end-to-end training through the pooled attention).
//
// A work item is the forward's: one 128-row query tile with its list of
// packed (KV block, level) segments, walked as 64-row KV sub-tiles.  The
// row log-sum-exp of the forward is known, so there is no running max:
//   p = 2^(s * sm_scale * log2 e + l - lse2),  ds = p (dp - D),
//   dQ = sm_scale * sum ds K^l.
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer: Q and dO tiles per item; per sub-tile one box
//               per (segment, 64-channel chunk) of the level-l K and V maps
//               into one ring stage, and the sub-tile record (attn_common.cuh).
//   warp 1      tcgen05 issuer: S_j = Q K_j^T and dP_j = dO V_j^T (M 128,
//               N 64) into double-buffered TMEM, then dQ += dS_{j-1} K_{j-1}
//               with dS read from TMEM (A) and K from shared memory (B,
//               MN-major), so S_{j+1} / dP_{j+1} run while the softmax
//               warpgroup works on sub-tile j.
//   warps 2..9  two warps per query row quarter, each on 32 of a sub-tile's
//               64 columns: p and ds, ds as bf16 into the S buffer; the
//               epilogue writes dQ * sm_scale, each warp half of the row.
// TMEM (512 columns): S at [0, 128), dP at [128, 256), dQ at [256, 256 + d).
// dS overwrites S in place: the packed bf16 pairs of columns 32 c .. 32 c + 31
// of a sub-tile go to columns 32 c .. 32 c + 15, written by the warp that
// read them.
// Every wait is bounded; a time-out sets the workspace status word.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "attn_common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kSoftWarps = 8;                       // two per TMEM lane quarter
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kThreads = 64 + kSoftThreads;
constexpr int kSub = kSubRows;

struct DqMaps {
  CUtensorMap m[10];
};

template <int NST>
struct DqShared {
  uint64_t q_full, q_empty;
  uint64_t kv_full[NST], kv_empty[NST];
  uint64_t i_full[NST], i_empty[NST];
  uint64_t s_full[2], ds_full[2];
  uint64_t o_final, o_free, drain;
  uint32_t tmem_base;
  int abort;
  SubInfo ti[NST];
};

__device__ __forceinline__ uint32_t sub_count(int rows) { return static_cast<uint32_t>((rows + kSub - 1) / kSub); }

template <int D, int NST, bool H2>
__global__ void __launch_bounds__(kThreads, 1) dq_kernel(const __grid_constant__ DqMaps maps, const DqArgs a) {
  constexpr int QB = D * 256;          // bytes of a 128-row tile
  constexpr int SB = D * 128;          // bytes of a 64-row K or V stage
  constexpr int KC = D / 64;
  constexpr uint32_t kTmemCols = 512;
  using Shared = DqShared<NST>;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sG = sQ + QB;               // dO
  uint8_t* sK = sG + QB;               // NST stages
  uint8_t* sV = sK + NST * SB;         // NST stages
  Shared* sh = reinterpret_cast<Shared*>(sV + NST * SB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = a.levels;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->q_full), 1);
    mbar_init(smem_u32(&sh->q_empty), 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(smem_u32(&sh->kv_full[i]), 1);
      mbar_init(smem_u32(&sh->kv_empty[i]), 1);
      mbar_init(smem_u32(&sh->i_full[i]), 32);
      mbar_init(smem_u32(&sh->i_empty[i]), kSoftThreads);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh->s_full[i]), 1);
      mbar_init(smem_u32(&sh->ds_full[i]), kSoftThreads);
    }
    mbar_init(smem_u32(&sh->o_final), 1);
    mbar_init(smem_u32(&sh->o_free), kSoftThreads);
    mbar_init(smem_u32(&sh->drain), 1);
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&sh->tmem_base), kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t tS = tmem, tP = tmem + 128, tQ = tmem + 256;
  volatile int* abort = &sh->abort;

  if (warp == 0) {
    // =============================== producer ===============================
    if (lane == 0) {
      for (int i = 0; i < 2 + 2 * L; ++i) tma_prefetch_desc(&maps.m[i]);
    }
    uint32_t it = 0, qcnt = 0, kvis = 0;
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
      if (!warp_wait(smem_u32(&sh->q_empty), (qcnt & 1) ^ 1, abort, a.status, 71, idx, qcnt, it, 0)) { ok = false; break; }
      if (lane == 0) {
        const uint32_t bar = smem_u32(&sh->q_full);
        mbar_arrive_expect_tx(bar, 2 * QB);
#pragma unroll
        for (int kc = 0; kc < KC; ++kc) {
          tma_load_3d(smem_u32(sQ + kc * 16384), &maps.m[0], bar, kc * 64, q0, bh);
          tma_load_3d(smem_u32(sG + kc * 16384), &maps.m[1], bar, kc * 64, q0, bh);
        }
      }
      ++qcnt;
      int sb = a.tile_seg_off[t0], nseg = a.tile_seg_off[t0 + 1] - sb;
      int w = lane < nseg ? a.segs[sb + lane] : 0;
      int nb = 0, nn = 0, wn = 0;
      int l = 0, half = 0, J = 0, rows = 0, r = 0;
      for (uint32_t j = 0; j < nsub && ok; ++j, ++it) {
        const int t = t0 + static_cast<int>(j >> 1);
        const int hs = static_cast<int>(j & 1);
        if (hs == 0) {
          if (j > 0) { sb = nb; nseg = nn; w = wn; }
          l = seg_level(w); half = seg_half(w); J = seg_block(w);
          rows = lane < nseg ? (a.block >> l) : 0;
          r = rows;
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
        bool mine;
        int lo, dst, cnt;
        if (rows > kSub) { mine = lane < nseg; lo = hs * kSub; dst = 0; cnt = kSub; }
        else { mine = lane < nseg && (r >> 6) == hs; lo = 0; dst = r - hs * kSub; cnt = rows; }
        const int prow = (half ? J * rows : nl) + lo;   // padding reads past the end: zeros
        const int st = it % NST;
        const uint32_t ph = (it / NST) & 1;

        // K and V of this sub-tile
        if (!warp_wait(smem_u32(&sh->kv_empty[st]), ph ^ 1, abort, a.status, 72, idx, j, it, 0)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(smem_u32(&sh->kv_full[st]), 2 * SB);
        __syncwarp();
        if (mine) {
#pragma unroll
          for (int kc = 0; kc < KC; ++kc) {
            tma_load_3d(smem_u32(sK + st * SB + kc * 8192 + dst * 128), &maps.m[2 + l], smem_u32(&sh->kv_full[st]),
                        kc * 64, prow, hkv);
            tma_load_3d(smem_u32(sV + st * SB + kc * 8192 + dst * 128), &maps.m[2 + L + l],
                        smem_u32(&sh->kv_full[st]), kc * 64, prow, hkv);
          }
        }
        ++kvis;
        // sub-tile record
        if (!warp_wait(smem_u32(&sh->i_empty[st]), ph ^ 1, abort, a.status, 73, idx, j, it, 0)) { ok = false; break; }
        write_subinfo<H2>(sh->ti[st], lane, mine, half, l, J, rows, lo, cnt, dst, w, nseg, nl, q0, a.N, a.block,
                          a.causal);
        mbar_arrive(smem_u32(&sh->i_full[st]));
      }
    }
    // drain: every copy this warp issued must land before the CTA exits
    if (lane == 0) {
      if (qcnt > 0) drain_wait(smem_u32(&sh->q_full), (qcnt - 1) & 1, a.status);
      for (uint32_t st = 0; st < static_cast<uint32_t>(NST); ++st)
        if (kvis > st) drain_wait(smem_u32(&sh->kv_full[st]), ((kvis - 1 - st) / NST) & 1, a.status);
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, kSub, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
      const uint64_t dQd = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dGd = sdesc_sw128(smem_u32(sG), 16, 1024);
      const uint64_t dKd = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dVd = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dKm = sdesc_sw128(smem_u32(sK), 8192, 1024);   // K as the MN-major B of dQ
      uint32_t it = 0, qcnt = 0, icnt = 0;
      bool ok = true;
      auto issue_dq = [&](uint32_t jj) -> bool {
        const uint32_t g = it + jj, st = g % NST, sb2 = g & 1;
        if (jj == 0 && icnt > 0) {
          if (!bounded_wait(smem_u32(&sh->o_free), (icnt - 1) & 1, abort, a.status, 81, icnt, jj, g, 0)) return false;
        }
        if (!bounded_wait(smem_u32(&sh->ds_full[sb2]), (g >> 1) & 1, abort, a.status, 82, icnt, jj, g, 0)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kSub / 16; ++k)
          // packed dS of columns 32 c .. 32 c + 31 sits at columns 32 c .. 32 c + 15
          umma_ts(tQ, tS + sb2 * kSub + k * 8 + (k >> 1) * 16, dKm + ((st * SB + k * 2048) >> 4), idO,
                  (jj == 0 && k == 0) ? 0u : 1u);
        umma_commit(smem_u32(&sh->kv_empty[st]));
        return true;
      };
      for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
        const int item = a.queue[idx];
        const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
        if (t1 == t0) continue;
        const uint32_t n = sub_count(a.item_rows[item]);
        if (!bounded_wait(smem_u32(&sh->q_full), qcnt & 1, abort, a.status, 83, idx, qcnt, it, 0)) { ok = false; break; }
        tc_fence_after();
        ++qcnt;
        for (uint32_t j = 0; j < n && ok; ++j) {
          const uint32_t g = it + j, st = g % NST, sb2 = g & 1;
          if (!bounded_wait(smem_u32(&sh->kv_full[st]), (g / NST) & 1, abort, a.status, 84, idx, j, g, 0)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t ao = (kc * 16384 + 32 * k) >> 4;
              const uint32_t bo = (st * SB + kc * 8192 + 32 * k) >> 4;
              umma_ss(tS + sb2 * kSub, dQd + ao, dKd + bo, idS, (kc | k) != 0);
              umma_ss(tP + sb2 * kSub, dGd + ao, dVd + bo, idS, (kc | k) != 0);
            }
          }
          umma_commit(smem_u32(&sh->s_full[sb2]));
          if (j + 1 == n) umma_commit(smem_u32(&sh->q_empty));
          if (j >= 1 && !issue_dq(j - 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_dq(n - 1)) { ok = false; break; }
        umma_commit(smem_u32(&sh->o_final));
        it += n;
        ++icnt;
      }
      umma_commit(smem_u32(&sh->drain));
      drain_wait(smem_u32(&sh->drain), 0, a.status);
    }
  } else {
    // =============================== softmax / epilogue ===============================
    const int q = warp & 3;
    const int cg = (warp - 2) >> 2;                       // 32-column group of each sub-tile
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int my_half = H2 ? (row >> 6) : 0;
    constexpr int DH = D / 2;                             // dQ columns this warp writes
    uint32_t it = 0, icnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
      const int item = a.queue[idx];
      const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
      const int bh = item / a.n_qtiles, tq = item - bh * a.n_qtiles;
      const int tok = tq * 128 + row;
      const int64_t orow = static_cast<int64_t>(bh) * a.N + tok;
      __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(a.dq) + orow * D + cg * DH;
      if (t1 == t0) {
        if (tok < a.N) {
          uint4* o = reinterpret_cast<uint4*>(dq);
          for (int c = 0; c < DH / 8; ++c) o[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const int64_t prow = (static_cast<int64_t>(bh) * a.n_qtiles + tq) * 128 + row;
      const float lse2 = a.lse2p[prow];
      const float Dv = a.dp[prow];
      const uint32_t n = sub_count(a.item_rows[item]);
      for (uint32_t j = 0; j < n; ++j, ++it) {
        const uint32_t st = it % NST, sb2 = it & 1;
        if (!warp_wait(smem_u32(&sh->s_full[sb2]), (it >> 1) & 1, abort, a.status, 91, idx, j, it, 0)) { ok = false; break; }
        if (!warp_wait(smem_u32(&sh->i_full[st]), (it / NST) & 1, abort, a.status, 92, idx, j, it, 0)) { ok = false; break; }
        tc_fence_after();
        const SubInfo& ti = sh->ti[st];
        uint32_t sr[32], dr[32];
        tmem_ld32(tS + sb2 * kSub + cg * 32 + lane_off, sr);
        tmem_ld32(tP + sb2 * kSub + cg * 32 + lane_off, dr);
        // exp2 argument of every column: s * sc + level - lse2 (or -inf)
        float x[32];
        const float sc = a.scale_log2;
        if (ti.fast) {
          const float cb0 = ti.cb[my_half][2 * cg] - lse2, cb1 = ti.cb[my_half][2 * cg + 1] - lse2;
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = fmaf(__uint_as_float(sr[c]), sc, c < 16 ? cb0 : cb1);
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 bv = *reinterpret_cast<const float4*>(&ti.bias[my_half][32 * cg + 4 * c4]);
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) x[4 * c4 + u] = fmaf(__uint_as_float(sr[4 * c4 + u]), sc, bb[u] - lse2);
          }
          if (ti.causal_check) {
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              const int4 iv = *reinterpret_cast<const int4*>(&ti.info[32 * cg + 4 * c4]);
              const int ii[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) x[4 * c4 + u] = ii[u] > tok ? -CUDART_INF_F : x[4 * c4 + u];
            }
          }
        }
        mbar_arrive(smem_u32(&sh->i_empty[st]));
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = 2 * i;
          const float p0 = fast_exp2(x[c]), p1 = fast_exp2(x[c + 1]);
          pk[i] = pack_bf16(p0 * (__uint_as_float(dr[c]) - Dv), p1 * (__uint_as_float(dr[c + 1]) - Dv));
        }
        // written over columns this warp read itself: its partner may not
        // have loaded its own columns yet
        tmem_st16(tS + sb2 * kSub + cg * 32 + lane_off, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->ds_full[sb2]));
      }
      if (!ok) break;
      if (!warp_wait(smem_u32(&sh->o_final), icnt & 1, abort, a.status, 93, idx, n, it, icnt)) { ok = false; break; }
      ++icnt;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tQ + cg * DH + c * 32 + lane_off, o);
        if (tok < a.N) {
          uint4* dst = reinterpret_cast<uint4*>(dq + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * a.sm_scale, __uint_as_float(o[8 * i + 1]) * a.sm_scale);
            v.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * a.sm_scale, __uint_as_float(o[8 * i + 3]) * a.sm_scale);
            v.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * a.sm_scale, __uint_as_float(o[8 * i + 5]) * a.sm_scale);
            v.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * a.sm_scale, __uint_as_float(o[8 * i + 7]) * a.sm_scale);
            dst[i] = v;
          }
        }
      }
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

template <int D, bool H2>
cudaError_t launch_q(const DqMaps& maps, const DqArgs& a, int num_sms, cudaStream_t s) {
  constexpr int NST = 4;
  const size_t smem = 1024 + 2 * static_cast<size_t>(D) * 256 + 2 * NST * static_cast<size_t>(D) * 128 +
                      sizeof(DqShared<NST>);
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(dq_kernel<D, NST, H2>), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dq_kernel<D, NST, H2><<<grid, kThreads, smem, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dq(const CUtensorMap* maps, const DqArgs& a, int num_sms, cudaStream_t s) {
  DqMaps m;
  for (int i = 0; i < 2 + 2 * a.levels; ++i) m.m[i] = maps[i];
  for (int i = 2 + 2 * a.levels; i < 10; ++i) m.m[i] = maps[0];
  if (a.d == 128) return a.block == 64 ? launch_q<128, true>(m, a, num_sms, s) : launch_q<128, false>(m, a, num_sms, s);
  return a.block == 64 ? launch_q<64, true>(m, a, num_sms, s) : launch_q<64, false>(m, a, num_sms, s);
}

}  // namespace psa
