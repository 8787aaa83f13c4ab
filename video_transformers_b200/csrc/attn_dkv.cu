// attn_dkv.cu -- dK and dV of adaptive pyramid attention, KV-major (the
// derivative of the forward of the summary article "PSA: Pyramid Sparse
// Attention ...", Method, with the mask held fixed; news review,
// Methodology 4: end-to-end training through the pooled attention).
//
// A work item is a 128-row tile of one pyramid level l of one KV head:
// pooled rows [128 t, 128 t + 128) of K^l and V^l, kept in shared memory.
// Its entries (from the transposed plan) are the query tiles that use some
// block of the tile at level l.  One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer: the K^l / V^l tile once per item; per entry
//               and 64-row query half, the Q and dO rows and the padded
//               lse2 / D values into a four-slot ring of half-tiles (a slot
//               is freed as soon as its half is accumulated, so the next
//               loads start a half-step earlier than with whole tiles).
//   warp 1      tcgen05 issuer (one thread), per 64-column query half hf:
//               S^T = K Q_hf^T and dP^T = V dO_hf^T (M 128 KV rows, N 64,
//               both operands from shared memory) into TMEM, then, once the
//               softmax has turned them into P^T and dS^T (bf16, in place),
//               dV += P^T dO_hf and dK += dS^T Q_hf with A read from TMEM
//               (M 128, N = d).  Half hf of an entry is accumulated before
//               the next entry's S^T of the same half is issued.
//   warps 2..9  two warps per KV row quarter, each on 32 of a half's 64
//               query columns: p = 2^(s * sm_scale * log2 e + l - lse2[q])
//               (0 when the row's block is not at level l for this query
//               half, or the pooled token is after the query under causal
//               masking), ds = p (dp - D[q]); then the epilogue writes the
//               item's dV^l (warps 2..5) and dK^l times sm_scale (warps
//               6..9) rows in fp32.
// TMEM (512 columns): S^T halves at [0, 64) and [64, 128), dP^T halves at
// [128, 256), dV at [256, 256 + d), dK at [256 + d, 256 + 2 d).  P^T and
// dS^T overwrite S^T and dP^T in place: the packed bf16 pairs of query
// columns 32 c .. 32 c + 31 go to buffer columns 32 c .. 32 c + 15, written by
// the warp that read those columns.
// Every wait is bounded; a time-out sets the workspace status word.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kSoftWarps = 8;                       // two per TMEM lane quarter
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kThreads = 64 + kSoftThreads;

struct DkvMaps {
  CUtensorMap m[10];
};

constexpr int kSlots = 4;     // query half-tiles in flight

struct DkvShared {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[kSlots], q_empty[kSlots];
  uint64_t s_full[2], p_full[2];
  uint64_t acc_full, acc_free, drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float lse2[kSlots][64];
  alignas(16) float dd[kSlots][64];
};

__device__ __forceinline__ void item_of(const DkvArgs& a, int item, int& l, int& b, int& hkv, int& t) {
  l = 0;
  while (item >= a.level_base[l + 1]) ++l;
  const int local = item - a.level_base[l];
  const int bhkv = local / a.level_tiles[l];
  t = local - bhkv * a.level_tiles[l];
  b = bhkv / a.Hkv;
  hkv = bhkv - b * a.Hkv;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) dkv_kernel(const __grid_constant__ DkvMaps maps, const DkvArgs a) {
  constexpr int TB = D * 256;          // bytes of a 128-row tile (K or V)
  constexpr int HB = D * 128;          // bytes of a 64-row half-tile (Q or dO)
  constexpr int KC = D / 64;           // 64-channel chunks
  constexpr uint32_t kTmemCols = 512;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = sK + TB;
  uint8_t* sQ = sV + TB;               // kSlots half-tiles
  uint8_t* sG = sQ + kSlots * HB;      // dO, kSlots half-tiles
  DkvShared* sh = reinterpret_cast<DkvShared*>(sG + kSlots * HB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = a.levels;
  const int grp = a.Hq / a.Hkv;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->kv_full), 1);
    mbar_init(smem_u32(&sh->kv_empty), 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(smem_u32(&sh->q_full[i]), 1);
      mbar_init(smem_u32(&sh->q_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh->s_full[i]), 1);
      mbar_init(smem_u32(&sh->p_full[i]), kSoftThreads);
    }
    mbar_init(smem_u32(&sh->acc_full), 1);
    mbar_init(smem_u32(&sh->acc_free), kSoftThreads);
    mbar_init(smem_u32(&sh->drain), 1);
    sh->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&sh->tmem_base), kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t tS = tmem, tP = tmem + 128, tV = tmem + 256, tK = tmem + 256 + D;
  volatile int* abort = &sh->abort;

  if (warp == 0) {
    // =============================== producer ===============================
    if (lane == 0) {
      for (int i = 0; i < 2 + 2 * L; ++i) tma_prefetch_desc(&maps.m[i]);
      uint32_t kcnt = 0, qiss = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
        const int item = a.n_items - 1 - idx;          // coarse levels (longest entry lists) first
        const int e0 = a.item_off[item], ne = a.item_off[item + 1] - e0;
        if (ne == 0) continue;
        int l, b, hkv, t;
        item_of(a, item, l, b, hkv, t);
        const int bhkv = b * a.Hkv + hkv;
        if (!bounded_wait(smem_u32(&sh->kv_empty), (kcnt & 1) ^ 1, abort, a.status, 41, idx, kcnt, 0, 0)) { ok = false; break; }
        const uint32_t kvb = smem_u32(&sh->kv_full);
        mbar_arrive_expect_tx(kvb, 2 * TB);
#pragma unroll
        for (int kc = 0; kc < KC; ++kc) {
          tma_load_3d(smem_u32(sK + kc * 16384), &maps.m[2 + l], kvb, kc * 64, t * 128, bhkv);
          tma_load_3d(smem_u32(sV + kc * 16384), &maps.m[2 + L + l], kvb, kc * 64, t * 128, bhkv);
        }
        ++kcnt;
        for (int e = 0; e < ne && ok; ++e) {
          const int qt = a.entry_qt[e0 + e];
          const int hl = qt / a.n_qtiles, tq = qt - hl * a.n_qtiles;
          const int bhq = b * a.Hq + hkv * grp + hl;
          for (int hf = 0; hf < 2; ++hf, ++qiss) {
            const uint32_t sl = qiss % kSlots, ph = (qiss / kSlots) & 1;
            if (!bounded_wait(smem_u32(&sh->q_empty[sl]), ph ^ 1, abort, a.status, 42, idx, e, qiss, hf)) { ok = false; break; }
            const uint32_t qb = smem_u32(&sh->q_full[sl]);
            mbar_arrive_expect_tx(qb, 2 * HB + 2 * 256);
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
              tma_load_3d(smem_u32(sQ + sl * HB + kc * 8192), &maps.m[0], qb, kc * 64, tq * 128 + hf * 64, bhq);
              tma_load_3d(smem_u32(sG + sl * HB + kc * 8192), &maps.m[1], qb, kc * 64, tq * 128 + hf * 64, bhq);
            }
            const int64_t prow = (static_cast<int64_t>(bhq) * a.n_qtiles + tq) * 128 + hf * 64;
            bulk_load(smem_u32(&sh->lse2[sl][0]), a.lse2p + prow, 256, qb);
            bulk_load(smem_u32(&sh->dd[sl][0]), a.dp + prow, 256, qb);
          }
        }
      }
      // drain: every copy issued must land before the CTA exits (the last
      // half loaded into slot sl is number qiss - 1 - ((qiss - 1 - sl) % kSlots))
      if (kcnt > 0) drain_wait(smem_u32(&sh->kv_full), (kcnt - 1) & 1, a.status);
      for (uint32_t sl = 0; sl < static_cast<uint32_t>(kSlots); ++sl)
        if (qiss > sl) drain_wait(smem_u32(&sh->q_full[sl]), ((qiss - 1 - sl) / kSlots) & 1, a.status);
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idA = idesc_bf16_f32(128, D, true);
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024);       // Q half as the K-major B of S^T
      const uint64_t dGk = sdesc_sw128(smem_u32(sG), 16, 1024);       // dO half as the K-major B of dP^T
      const uint64_t dQm = sdesc_sw128(smem_u32(sQ), 8192, 1024);     // Q half as the MN-major B of dK
      const uint64_t dGm = sdesc_sw128(smem_u32(sG), 8192, 1024);     // dO half as the MN-major B of dV
      uint32_t kcnt = 0, u = 0;        // u: query halves consumed (slot u % kSlots)
      bool ok = true;
      // dV += P^T dO_h, dK += dS^T Q_h for half number uh (TMEM buffers hf = uh & 1),
      // then its slot is released
      auto accumulate = [&](uint32_t uh, bool first) -> bool {
        const int hf = uh & 1;
        if (!bounded_wait(smem_u32(&sh->p_full[hf]), (uh >> 1) & 1, abort, a.status, 52, uh, hf, 0, 0)) return false;
        tc_fence_after();
        const uint32_t sl = uh % kSlots;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t off = (sl * HB + k * 2048) >> 4;
          const uint32_t acc = (first && k == 0) ? 0u : 1u;
          // the packed P^T / dS^T of query columns 32 cg .. 32 cg + 31 sit at
          // TMEM columns 32 cg .. 32 cg + 15 of the buffer (see the softmax)
          const uint32_t ac = hf * 64 + k * 8 + (k >> 1) * 16;
          umma_ts(tV, tS + ac, dGm + off, idA, acc);
          umma_ts(tK, tP + ac, dQm + off, idA, acc);
        }
        umma_commit(smem_u32(&sh->q_empty[sl]));
        return true;
      };
      for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
        const int item = a.n_items - 1 - idx;
        const int ne = a.item_off[item + 1] - a.item_off[item];
        if (ne == 0) continue;
        if (!bounded_wait(smem_u32(&sh->kv_full), kcnt & 1, abort, a.status, 51, idx, kcnt, 0, 0)) { ok = false; break; }
        if (kcnt > 0 && !bounded_wait(smem_u32(&sh->acc_free), (kcnt - 1) & 1, abort, a.status, 53, idx, kcnt, 0, 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t u0 = u;
        for (int e = 0; e < ne && ok; ++e) {
          for (int hf = 0; hf < 2; ++hf, ++u) {
            // the previous entry's half hf frees TMEM buffer hf before S^T of this one
            if (e > 0 && !accumulate(u - 2, u - 2 == u0)) { ok = false; break; }
            const uint32_t sl = u % kSlots;
            if (!bounded_wait(smem_u32(&sh->q_full[sl]), (u / kSlots) & 1, abort, a.status, 54, idx, e, u, 0)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t ao = (kc * 16384 + 32 * k) >> 4;
                const uint32_t bo = (sl * HB + kc * 8192 + 32 * k) >> 4;
                umma_ss(tS + hf * 64, dK + ao, dQk + bo, idS, (kc | k) != 0);
                umma_ss(tP + hf * 64, dV + ao, dGk + bo, idS, (kc | k) != 0);
              }
            }
            umma_commit(smem_u32(&sh->s_full[hf]));
          }
        }
        if (!ok) break;
        for (int hf = 0; hf < 2; ++hf)
          if (!accumulate(u - 2 + hf, u - 2 + hf == u0)) { ok = false; break; }
        if (!ok) break;
        umma_commit(smem_u32(&sh->acc_full));
        umma_commit(smem_u32(&sh->kv_empty));
        ++kcnt;
      }
      umma_commit(smem_u32(&sh->drain));
      drain_wait(smem_u32(&sh->drain), 0, a.status);
    }
  } else {
    // =============================== softmax / epilogue ===============================
    const int q = warp & 3;
    const int cg = (warp - 2) >> 2;                       // 32-column group of each half
    const int r = q * 32 + lane;                          // KV row of the tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t kcnt = 0, g = 0;        // g: entries processed (query halves 2 g, 2 g + 1)
    bool ok = true;
    for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
      const int item = a.n_items - 1 - idx;
      const int e0 = a.item_off[item], ne = a.item_off[item + 1] - e0;
      int l, b, hkv, t;
      item_of(a, item, l, b, hkv, t);
      const int Nl = a.N >> l;
      const int p = t * 128 + r;                          // pooled row of level l
      const bool row_in = p < Nl;
      const int jb = r / (a.block >> l);                  // block of the tile holding this row
      const int last_tok = ((p + 1) << l) - 1;            // last token the pooled row averages
      const float bias = static_cast<float>(l);           // ln 2^l in log2 units
      const int64_t orow = a.level_off[l] + (static_cast<int64_t>(b * a.Hkv + hkv) * Nl + p) * D;
      float* gout = cg == 0 ? a.dvl : a.dkl;
      const float oscale = cg == 0 ? 1.0f : a.sm_scale;
      if (ne == 0) {
        if (row_in) {
          float4* o4 = reinterpret_cast<float4*>(gout + orow);
          for (int c = 0; c < D / 4; ++c) o4[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      for (int e = 0; e < ne && ok; ++e, ++g) {
        const unsigned bits = a.entry_mask[e0 + e];
        const int qt = a.entry_qt[e0 + e];
        const int tq = qt - (qt / a.n_qtiles) * a.n_qtiles;
        for (int hf = 0; hf < 2; ++hf) {
          if (!warp_wait(smem_u32(&sh->s_full[hf]), g & 1, abort, a.status, 61, idx, e, g, hf)) { ok = false; break; }
          tc_fence_after();
          uint32_t sr[32], dr[32];
          tmem_ld32(tS + hf * 64 + cg * 32 + lane_off, sr);
          tmem_ld32(tP + hf * 64 + cg * 32 + lane_off, dr);
          const bool valid = row_in && ((bits >> (2 * jb + hf)) & 1u);
          const int q_first = tq * 128 + hf * 64 + cg * 32;   // token of this thread's column 0
          // column c (query token q_first + c) sees the pooled row iff the
          // row is valid and, under causal masking, last_tok <= q_first + c:
          // the hidden columns are exactly c < cut
          const int cut = !valid ? 32 : (a.causal ? max(0, min(32, last_tok - q_first)) : 0);
          const float sc = a.scale_log2;
          const uint32_t sl = (2 * g + hf) % kSlots;
          const float4* lz4 = reinterpret_cast<const float4*>(&sh->lse2[sl][cg * 32]);
          const float4* dz4 = reinterpret_cast<const float4*>(&sh->dd[sl][cg * 32]);
          uint32_t pk[16], gk[16];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 lv = lz4[i4], dv = dz4[i4];
            const float lz[4] = {lv.x, lv.y, lv.z, lv.w}, dz[4] = {dv.x, dv.y, dv.z, dv.w};
            float pv[4], gv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = 4 * i4 + u;
              const float x = c < cut ? -CUDART_INF_F : fmaf(__uint_as_float(sr[c]), sc, bias - lz[u]);
              pv[u] = fast_exp2(x);
              gv[u] = pv[u] * (__uint_as_float(dr[c]) - dz[u]);
            }
            pk[2 * i4] = pack_bf16(pv[0], pv[1]);
            pk[2 * i4 + 1] = pack_bf16(pv[2], pv[3]);
            gk[2 * i4] = pack_bf16(gv[0], gv[1]);
            gk[2 * i4 + 1] = pack_bf16(gv[2], gv[3]);
          }
          // each warp writes its packed half only over columns it has read
          // itself (its partner may not have loaded its own columns yet)
          tmem_st16(tS + hf * 64 + cg * 32 + lane_off, pk);
          tmem_st16(tP + hf * 64 + cg * 32 + lane_off, gk);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(smem_u32(&sh->p_full[hf]));
        }
      }
      if (!ok) break;
      // epilogue: warps of column group 0 write dV^l, group 1 dK^l (times sm_scale)
      if (!warp_wait(smem_u32(&sh->acc_full), kcnt & 1, abort, a.status, 62, idx, kcnt, 0, 0)) { ok = false; break; }
      ++kcnt;
      tc_fence_after();
      const uint32_t tacc = cg == 0 ? tV : tK;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tacc + c * 32 + lane_off, v);
        if (row_in) {
          float4* o4 = reinterpret_cast<float4*>(gout + orow + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o4[i] = make_float4(__uint_as_float(v[4 * i]) * oscale, __uint_as_float(v[4 * i + 1]) * oscale,
                                __uint_as_float(v[4 * i + 2]) * oscale, __uint_as_float(v[4 * i + 3]) * oscale);
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&sh->acc_free));
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

template <int D>
cudaError_t launch_d(const DkvMaps& maps, const DkvArgs& a, int num_sms, cudaStream_t s) {
  const size_t smem = 1024 + 2 * static_cast<size_t>(D) * 256 + 2 * kSlots * static_cast<size_t>(D) * 128 +
                      sizeof(DkvShared);
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(dkv_kernel<D>), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dkv_kernel<D><<<grid, kThreads, smem, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dkv(const CUtensorMap* maps, const DkvArgs& a, int num_sms, cudaStream_t s) {
  DkvMaps m;
  for (int i = 0; i < 2 + 2 * a.levels; ++i) m.m[i] = maps[i];
  for (int i = 2 + 2 * a.levels; i < 10; ++i) m.m[i] = maps[0];
  return a.d == 128 ? launch_d<128>(m, a, num_sms, s) : launch_d<64>(m, a, num_sms, s);
}

}  // namespace psa
