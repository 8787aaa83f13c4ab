// attn.cu -- stage 3 of the PSA forward path: adaptive pyramid attention
// (summary article "PSA: Pyramid Sparse Attention ...", Method: every KV
// block is read at the pyramid level the mask assigns it and a scale factor
// keeps the probabilities consistent; the kernel separates the logical block
// size from the hardware tile size; news review, Methodology 4: ordinary
// scaled dot-product attention over the pooled KV).
//
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer: Q of the work item, then per 128-row KV tile one
//               box per (segment, 64-channel chunk) of the level-l K and V
//               maps, plus a per-column record (level bias, validity, last
//               covered token, query-half mask) written to shared memory.
//   warp 1      tcgen05 issuer (one thread): S = Q K^T into one of two TMEM
//               S buffers, O += P V with P read from TMEM.
//   warps 2..5  softmax, one query row per thread: S from TMEM, logit
//               z = s * scale * log2(e) + l (the +ln 2^l bias in log2 units),
//               online max / sum with lazy rescaling of O, P (bf16) back into
//               the S buffer, and the final O / l and lse store.
// Every wait is bounded; a time-out sets the workspace status word.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "sm100.cuh"

namespace psa {
namespace {

constexpr int kThreads = 192;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 256

struct AttnMaps {
  CUtensorMap m[9];
};

template <int NST>
struct AttnShared {
  uint64_t q_full, q_empty;
  uint64_t kv_full[NST], kv_empty[NST];
  uint64_t s_full[2], p_full[2];
  uint64_t o_ready, o_final, o_free, drain;
  uint32_t tmem_base;
  int abort;
  int flags[NST];
  float bias[NST][128];
  int info[NST][128];   // (last covered token << 2) | query-half mask
};

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  constexpr int NST = D == 128 ? 2 : 4;
  constexpr int QB = D * 256;          // bytes of a 128-row tile of D bf16 channels
  constexpr int KC = D / 64;           // 64-channel chunks
  using Shared = AttnShared<NST>;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + QB;
  uint8_t* sV = sK + NST * QB;
  Shared* sh = reinterpret_cast<Shared*>(sV + NST * QB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = a.levels;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sh->q_full), 1);
    mbar_init(smem_u32(&sh->q_empty), 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(smem_u32(&sh->kv_full[i]), 32);
      mbar_init(smem_u32(&sh->kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh->s_full[i]), 1);
      mbar_init(smem_u32(&sh->p_full[i]), 128);
    }
    mbar_init(smem_u32(&sh->o_ready), 1);
    mbar_init(smem_u32(&sh->o_final), 1);
    mbar_init(smem_u32(&sh->o_free), 128);
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

  if (warp == 0) {
    // =============================== producer ===============================
    if (lane == 0) {
      for (int i = 0; i < 1 + 2 * L; ++i) tma_prefetch_desc(&maps.m[i]);
    }
    uint32_t kv_it = 0, qcnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
      const int item = a.queue[idx];
      const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
      if (t1 == t0) continue;
      const int bh = item / a.n_qtiles, tq = item - bh * a.n_qtiles;
      const int b = bh / a.Hq, h = bh - b * a.Hq;
      const int hkv = b * a.Hkv + h / (a.Hq / a.Hkv);
      const int q0 = tq * 128;
      if (!warp_wait(smem_u32(&sh->q_empty), (qcnt & 1) ^ 1, abort, a.status, 11, idx, qcnt, kv_it, 0)) { ok = false; break; }
      if (lane == 0) {
        const uint32_t bar = smem_u32(&sh->q_full);
        mbar_arrive_expect_tx(bar, QB);
#pragma unroll
        for (int kc = 0; kc < KC; ++kc) tma_load_3d(smem_u32(sQ + kc * 16384), &maps.m[0], bar, kc * 64, q0, bh);
      }
      ++qcnt;
      for (int t = t0; t < t1; ++t, ++kv_it) {
        const int st = kv_it % NST;
        if (!warp_wait(smem_u32(&sh->kv_empty[st]), ((kv_it / NST) & 1) ^ 1, abort, a.status, 12, idx, t - t0, kv_it, 0)) { ok = false; break; }
        const int sb = a.tile_seg_off[t], se = a.tile_seg_off[t + 1];
        const uint32_t bar = smem_u32(&sh->kv_full[st]);
        if (lane == 0) {
          mbar_expect_tx(bar, 2 * QB);
          const uint32_t dK = smem_u32(sK + st * QB), dV = smem_u32(sV + st * QB);
          int r = 0;
          for (int s = sb; s < se; ++s) {
            const int w = a.segs[s];
            const int l = seg_level(w), half = seg_half(w), J = seg_block(w);
            const int rows = a.block >> l;
            const int prow = half ? J * rows : (a.N >> l);   // padding reads past the end: zeros
#pragma unroll
            for (int kc = 0; kc < KC; ++kc) {
              tma_load_3d(dK + kc * 16384 + r * 128, &maps.m[1 + l], bar, kc * 64, prow, hkv);
              tma_load_3d(dV + kc * 16384 + r * 128, &maps.m[1 + L + l], bar, kc * 64, prow, hkv);
            }
            r += rows;
          }
        }
        // per-column record of this tile
        bool need = false;
        int r = 0;
        for (int s = sb; s < se; ++s) {
          const int w = a.segs[s];
          const int l = seg_level(w), half = seg_half(w), J = seg_block(w);
          const int rows = a.block >> l;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int c = lane + 32 * m;
            if (c >= r && c < r + rows) {
              const int p = J * rows + (c - r);
              const bool valid = half != 0 && p < (a.N >> l);
              const int last = ((p + 1) << l) - 1;
              sh->bias[st][c] = valid ? static_cast<float>(l) : -CUDART_INF_F;
              sh->info[st][c] = (last << 2) | half;
              need |= valid && (half != 3 || (a.causal && last > q0));
            }
          }
          r += rows;
        }
        const bool any = __any_sync(0xffffffffu, need);
        if (lane == 0) sh->flags[st] = any ? 1 : 0;
        __syncwarp();
        mbar_arrive(bar);
      }
    }
    // drain: wait for every TMA this warp issued before the CTA may exit
    if (lane == 0) {
      if (qcnt > 0) drain_wait(smem_u32(&sh->q_full), (qcnt - 1) & 1, a.status);
      for (uint32_t st = 0; st < NST; ++st) {
        if (kv_it > st) drain_wait(smem_u32(&sh->kv_full[st]), ((kv_it - 1 - st) / NST) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // =============================== MMA issuer ===============================
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, true);
      const uint32_t tO = tmem + 256;
      uint32_t kv_it = 0, T = 0, qcnt = 0, icnt = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t jj, bool first_of_item) -> bool {
        const uint32_t st = (kv_it + jj) % NST;
        const uint32_t buf = (T + jj) & 1;
        if (first_of_item && icnt > 0) {
          if (!bounded_wait(smem_u32(&sh->o_free), (icnt - 1) & 1, abort, a.status, 21, icnt, jj, T, kv_it)) return false;
        }
        if (!bounded_wait(smem_u32(&sh->p_full[buf]), ((T + jj) >> 1) & 1, abort, a.status, 22, icnt, jj, T, kv_it)) return false;
        tc_fence_after();
        const uint32_t sV_st = smem_u32(sV + st * QB);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          umma_ts(tO, tmem + buf * 128 + k * 8, sdesc_sw128(sV_st + k * 2048, 16384, 1024), idO,
                  (first_of_item && k == 0) ? 0u : 1u);
        }
        umma_commit(smem_u32(&sh->kv_empty[st]));
        umma_commit(smem_u32(&sh->o_ready));
        return true;
      };
      for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
        const int item = a.queue[idx];
        const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
        const uint32_t n = static_cast<uint32_t>(t1 - t0);
        if (n == 0) continue;
        if (!bounded_wait(smem_u32(&sh->q_full), qcnt & 1, abort, a.status, 23, idx, qcnt, T, kv_it)) { ok = false; break; }
        tc_fence_after();
        ++qcnt;
        const uint32_t sQb = smem_u32(sQ);
        for (uint32_t j = 0; j < n && ok; ++j) {
          const uint32_t st = (kv_it + j) % NST;
          const uint32_t buf = (T + j) & 1;
          if (!bounded_wait(smem_u32(&sh->kv_full[st]), ((kv_it + j) / NST) & 1, abort, a.status, 24, idx, j, T, kv_it)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sK_st = smem_u32(sK + st * QB);
#pragma unroll
          for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              umma_ss(tmem + buf * 128, sdesc_sw128(sQb + kc * 16384 + 32 * k, 16, 1024),
                      sdesc_sw128(sK_st + kc * 16384 + 32 * k, 16, 1024), idS, (kc | k) != 0);
            }
          }
          umma_commit(smem_u32(&sh->s_full[buf]));
          if (j + 1 == n) umma_commit(smem_u32(&sh->q_empty));
          if (j >= 1) {
            if (!issue_pv(j - 1, j == 1)) { ok = false; break; }
          }
        }
        if (!ok) break;
        if (!issue_pv(n - 1, n == 1)) { ok = false; break; }
        umma_commit(smem_u32(&sh->o_final));   // O of this item is complete
        kv_it += n;
        T += n;
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
    const int my_half_bit = 1 << (row >> 6);
    uint32_t kv_it = 0, T = 0, pv = 0, icnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < a.n_items && ok; idx += gridDim.x) {
      const int item = a.queue[idx];
      const int t0 = a.item_tile_off[item], t1 = a.item_tile_off[item + 1];
      const int bh = item / a.n_qtiles, tq = item - bh * a.n_qtiles;
      const int tok = tq * 128 + row;
      const int64_t orow = static_cast<int64_t>(bh) * a.N + tok;
      const int n = t1 - t0;
      if (n == 0) {
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
      float m = -CUDART_INF_F, lsum = 0.f;
      for (int j = 0; j < n; ++j, ++kv_it, ++T, ++pv) {
        const int st = kv_it % NST;
        const int buf = T & 1;
        if (!warp_wait(smem_u32(&sh->s_full[buf]), (T >> 1) & 1, abort, a.status, 31, idx, j, T, kv_it)) { ok = false; break; }
        if (!warp_wait(smem_u32(&sh->kv_full[st]), (kv_it / NST) & 1, abort, a.status, 32, idx, j, T, kv_it)) { ok = false; break; }
        tc_fence_after();
        float s[128];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t raw[32];
          tmem_ld32(tmem + buf * 128 + c4 * 32 + lane_off, raw);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            s[c4 * 32 + i] = fmaf(__uint_as_float(raw[i]), a.scale_log2, sh->bias[st][c4 * 32 + i]);
        }
        if (sh->flags[st]) {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const int inf = sh->info[st][c];
            const bool vis = (inf & my_half_bit) && (!a.causal || (inf >> 2) <= tok);
            s[c] = vis ? s[c] : -CUDART_INF_F;
          }
        }
        float mt = s[0];
#pragma unroll
        for (int c = 1; c < 128; ++c) mt = fmaxf(mt, s[c]);
        const float mnew = fmaxf(m, mt);
        // Lazy rescaling: a row moves its reference max only when the new max
        // exceeds it by more than kRescaleThreshold (or on its first visible
        // key).  O lives in TMEM and is read/written with warp-collective
        // tcgen05.ld/st, so the decision to touch O is taken per warp.
        const bool first = m == -CUDART_INF_F && mnew != -CUDART_INF_F;
        const bool grow = m != -CUDART_INF_F && mnew > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
          const float f = grow ? fast_exp2(m - mnew) : 1.0f;
          lsum *= f;
          if (grow) m = mnew;
          // O holds tiles 0..j-1: wait for the PV of tile j-1, then scale it
          if (!warp_wait(smem_u32(&sh->o_ready), (pv - 1) & 1, abort, a.status, 33, idx, j, pv, 0)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + 256 + c * 32 + lane_off, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tmem + 256 + c * 32 + lane_off, o);
          }
        }
        if (first) m = mnew;
        const float mu = m == -CUDART_INF_F ? 0.f : m;
        float ps = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = fast_exp2(s[2 * i] - mu), p1 = fast_exp2(s[2 * i + 1] - mu);
          ps += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        lsum += ps;
        tmem_st32(tmem + buf * 128 + lane_off, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
        tmem_st32(tmem + buf * 128 + 32 + lane_off, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sh->p_full[buf]));
      }
      if (!ok) break;
      // epilogue: O / l, once the item's last PV is done (o_final completes
      // once per item; the MMA cannot start the next item's PVs before o_free,
      // so its phases never run two ahead of this wait)
      if (!warp_wait(smem_u32(&sh->o_final), icnt & 1, abort, a.status, 35, idx, n, pv, icnt)) { ok = false; break; }
      ++icnt;
      tc_fence_after();
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + 256 + c * 32 + lane_off, o);
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
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool F32>
cudaError_t launch_one(const AttnMaps& maps, const AttnArgs& a, int num_sms, cudaStream_t s) {
  constexpr int NST = D == 128 ? 2 : 4;
  const size_t smem = 1024 + static_cast<size_t>(D) * 256 * (1 + 2 * NST) + sizeof(AttnShared<NST>);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  attn_kernel<D, F32><<<grid, kThreads, smem, s>>>(maps, a);
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

}  // namespace psa
