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
//               the 128-row Q and dO tiles and the padded lse2 / D rows into
//               a two-stage ring.
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
// [128, 256), dV at [256, 256 + d), dK at [256 + d, 256 + 2 d).
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

struct DkvShared {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t acc_full, acc_free, drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float lse2[2][128];
  alignas(16) float dd[2][128];
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
  constexpr int TB = D * 256;          // bytes of a 128-row tile (K, V, Q or dO)
  constexpr int KC = D / 64;           // 64-channel chunks, 16 KB each
  constexpr uint32_t kTmemCols = 512;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = sK + TB;
  uint8_t* sQ = sV + TB;               // 2 stages
  uint8_t* sG = sQ + 2 * TB;           // dO, 2 stages
  DkvShared* sh = reinterpret_cast<DkvShared*>(sG + 2 * TB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = a.levels;
  const int grp = a.Hq / a.Hkv;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->kv_full), 1);
    mbar_init(smem_u32(&sh->kv_empty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh->q_full[i]), 1);
      mbar_init(smem_u32(&sh->q_empty[i]), 1);
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
        for (int e = 0; e < ne; ++e, ++qiss) {
          const uint32_t st = qiss & 1, ph = (qiss >> 1) & 1;
          if (!bounded_wait(smem_u32(&sh->q_empty[st]), ph ^ 1, abort, a.status, 42, idx, e, qiss, 0)) { ok = false; break; }
          const int qt = a.entry_qt[e0 + e];
          const int hl = qt / a.n_qtiles, tq = qt - hl * a.n_qtiles;
          const int bhq = b * a.Hq + hkv * grp + hl;
          const uint32_t qb = smem_u32(&sh->q_full[st]);
          mbar_arrive_expect_tx(qb, 2 * TB + 2 * 512);
#pragma unroll
          for (int kc = 0; kc < KC; ++kc) {
            tma_load_3d(smem_u32(sQ + st * TB + kc * 16384), &maps.m[0], qb, kc * 64, tq * 128, bhq);
            tma_load_3d(smem_u32(sG + st * TB + kc * 16384), &maps.m[1], qb, kc * 64, tq * 128, bhq);
          }
          const int64_t prow = (static_cast<int64_t>(bhq) * a.n_qtiles + tq) * 128;
          bulk_load(smem_u32(&sh->lse2[st][0]), a.lse2p + prow, 512, qb);
          bulk_load(smem_u32(&sh->dd[st][0]), a.dp + prow, 512, qb);
        }
      }
      // drain: every copy issued must land before the CTA exits
      if (kcnt > 0) drain_wait(smem_u32(&sh->kv_full), (kcnt - 1) & 1, a.status);
      for (uint32_t st = 0; st < 2; ++st)
        if (qiss > st) drain_wait(smem_u32(&sh->q_full[st]), ((qiss - 1 - st) / 2) & 1, a.status);
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idA = idesc_bf16_f32(128, D, true);
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024);       // Q as the K-major B of S^T
      const uint64_t dGk = sdesc_sw128(smem_u32(sG), 16, 1024);       // dO as the K-major B of dP^T
      const uint64_t dQm = sdesc_sw128(smem_u32(sQ), 16384, 1024);    // Q as the MN-major B of dK
      const uint64_t dGm = sdesc_sw128(smem_u32(sG), 16384, 1024);    // dO as the MN-major B of dV
      uint32_t kcnt = 0, g = 0;
      bool ok = true;
      // dV += P^T dO_hf, dK += dS^T Q_hf for entry number ge (stage ge & 1)
      auto accumulate = [&](uint32_t ge, int hf, bool first) -> bool {
        if (!bounded_wait(smem_u32(&sh->p_full[hf]), ge & 1, abort, a.status, 52, ge, hf, 0, 0)) return false;
        tc_fence_after();
        const uint32_t st = ge & 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t off = (st * TB + hf * 8192 + k * 2048) >> 4;
          const uint32_t acc = (first && k == 0) ? 0u : 1u;
          umma_ts(tV, tS + hf * 64 + k * 8, dGm + off, idA, acc);
          umma_ts(tK, tP + hf * 64 + k * 8, dQm + off, idA, acc);
        }
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
        const uint32_t g0 = g;
        for (int e = 0; e < ne && ok; ++e, ++g) {
          const uint32_t st = g & 1;
          if (!bounded_wait(smem_u32(&sh->q_full[st]), (g >> 1) & 1, abort, a.status, 54, idx, e, g, 0)) { ok = false; break; }
          tc_fence_after();
          for (int hf = 0; hf < 2; ++hf) {
            if (e > 0 && !accumulate(g - 1, hf, g - 1 == g0 && hf == 0)) { ok = false; break; }
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t ao = (kc * 16384 + 32 * k) >> 4;
                const uint32_t bo = (st * TB + kc * 16384 + hf * 8192 + 32 * k) >> 4;
                umma_ss(tS + hf * 64, dK + ao, dQk + bo, idS, (kc | k) != 0);
                umma_ss(tP + hf * 64, dV + ao, dGk + bo, idS, (kc | k) != 0);
              }
            }
            umma_commit(smem_u32(&sh->s_full[hf]));
          }
          if (!ok) break;
          if (e > 0) umma_commit(smem_u32(&sh->q_empty[(g - 1) & 1]));
        }
        if (!ok) break;
        for (int hf = 0; hf < 2; ++hf)
          if (!accumulate(g - 1, hf, g - 1 == g0 && hf == 0)) { ok = false; break; }
        if (!ok) break;
        umma_commit(smem_u32(&sh->q_empty[(g - 1) & 1]));
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
    uint32_t kcnt = 0, g = 0;
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
        const uint32_t st = g & 1;
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
          const float4* lz4 = reinterpret_cast<const float4*>(&sh->lse2[st][hf * 64 + cg * 32]);
          const float4* dz4 = reinterpret_cast<const float4*>(&sh->dd[st][hf * 64 + cg * 32]);
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
          tmem_st16(tS + hf * 64 + cg * 16 + lane_off, pk);
          tmem_st16(tP + hf * 64 + cg * 16 + lane_off, gk);
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
  const size_t smem = 1024 + 6 * static_cast<size_t>(D) * 256 + sizeof(DkvShared);
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
