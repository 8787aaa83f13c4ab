// internal.h -- declarations shared by the PSA library's translation units.
// Not part of the public ABI (include/psa.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/psa.h"

namespace psa {

// SM count of the current device, looked up once per device.
int device_sm_count();
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) of kernel `fn` on the
// current device, done once per (kernel, device) and remembered.
cudaError_t set_smem_limit(const void* fn, int bytes);

// 2^x for x <= 0 (a difference of log-sum-exps, log2 domain) with relative
// error about 2.5e-7: x = n + f with n = floor(x) in fp64, 2^f of the
// fraction rounded to fp32 from the special-function unit, 2^n applied to
// the exponent exactly.  Arguments below -1000 give 0.
__device__ __forceinline__ double exp2_split(double x) {
  if (x < -1000.0) return 0.0;
  const double n = floor(x);
  float p;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p) : "f"(static_cast<float>(x - n)));
  return ldexp(static_cast<double>(p), static_cast<int>(n));
}

// ---- stage 1 -------------------------------------------------------------
// Pools K and V ([BH, N, d], elem = 2 (bf16) or 4 (fp32)) into levels
// 1..L-1 written at the given byte offsets of k_pyr / v_pyr.
cudaError_t launch_pyramid(const void* k, const void* v, void* k_pyr, void* v_pyr, int64_t BH,
                           int N, int d, int levels, int elem, const size_t* level_off,
                           cudaStream_t s);
cudaError_t launch_blockcos(const void* k, float* out, int64_t BH, int N, int d, int block,
                            int elem, cudaStream_t s);
cudaError_t launch_cast_bf16(const float* src, void* dst, int64_t n, cudaStream_t s);

// ---- stage 2 -------------------------------------------------------------
// column parts of the paired sampling score (score2_kernel): a work item is
// (head, row-tile pair, part), and part e writes row-LSE partial e
constexpr int kScore2Parts = 4;

struct ScoreArgs {
  int BHq, Hq, Hkv, N, d, block, nkb;
  int mode;            // 0 sampling, 1 antidiagonal
  int step;            // token distance between rows of the A view (block/8 or S)
  int S;               // antidiagonal stride (1 for sampling)
  int rows;            // score rows per head (nqb*8 or N/S)
  int cols;            // score columns per head (N or N/S)
  int rows_per_block;  // 8 (sampling) or block/S
  int cols_per_block;  // block (sampling) or block/S
  int causal;
  float scale_log2;    // softmax scale * log2(e)
  float* blocklse;     // [BHq][nkb][rows]  log2-domain logsumexp of each block
  float* rowlse;       // [n_part][BHq][rows]  partial row LSEs (score_kernel: 2, one per epilogue
                       // warpgroup; score2_kernel: kScore2Parts, one per column part)
  int* status;
};
cudaError_t launch_score(const CUtensorMap* mapA, const CUtensorMap* mapB, const ScoreArgs& a,
                         int num_sms, cudaStream_t s);

// Mean-key scorer (mode 2): block means of Q and K in fp64, then one score
// row per query block written in the same [BHq][nkb][rows] / [2][BHq][rows]
// log2-domain layout the score kernel uses (rows = nqb, one row per block).
cudaError_t launch_blockmean(const void* x, double* out, int64_t BH, int N, int d, int block, int elem,
                             bool transpose, cudaStream_t s);
struct MeanKeyArgs {
  int BHq, Hq, Hkv, d, nqb, nkb, causal;
  double scale_log2;        // sm_scale * log2(e)
  const double* qmean;      // [BHq][d][nqb]
  const double* kmeanT;     // [BHkv][d][nkb]
  float* blocklse;          // [BHq][nkb][nqb]
  float* rowlse;            // [2][BHq][nqb]
};
cudaError_t launch_meankey_score(const MeanKeyArgs& a, cudaStream_t s);

struct SelectArgs {
  int B, Hq, Hkv, N, block, nqb, nkb, levels, causal;
  int mode, S, rows, rows_per_block, step;
  int policy;               // 0 levels by exclusive prefix of mass, 1 by rank / visible blocks
  float thresholds[8];
  float cos_min;
  int n_dense_prefix;
  const float* blocklse;
  const float* rowlse;      // [n_part][B*Hq][rows]
  int n_part;               // row-LSE partials to combine per row
  const float* blockcos;
  uint8_t* mask;
  float* mass_out;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);

// ---- stage 3 -------------------------------------------------------------
struct PlanArgs {
  int B, Hq, N, block, nqb, nkb, levels, causal;
  int n_items;           // query tiles of 128 rows: B*Hq*ceil(N/128)
  const uint8_t* mask;
  int* item_nseg;        // [n_items]   segments per item (pads included)
  int* item_ntile;       // [n_items]
  int* item_rows;        // [n_items]   real (non-padding) KV rows per item
  int* item_seg_off;     // [n_items+1]
  int* item_tile_off;    // [n_items+1]
  int* tile_seg_off;     // [max_tiles+1]
  int* segs;             // [max_segs]
  int* queue;            // [n_items]  item ids in processing order
  int lpt_queue;         // 1: most tiles first; 0: natural (head-major) order
  int* hist;             // [n_hist]   scratch for the counting sort
  int n_hist;
  long long* stats;      // [2] tiles, real kv rows
};
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s);

struct AttnArgs {
  int B, Hq, Hkv, N, d, block, levels, causal;
  int n_items, n_qtiles;  // n_qtiles = ceil(N/128) per head
  float scale_log2;       // sm_scale * log2(e)
  const int* item_tile_off;
  const int* item_rows;   // real KV rows per item (sub-tiles = ceil(rows / 64))
  const int* tile_seg_off;
  const int* segs;
  const int* queue;
  void* out;              // [B,Hq,N,d] bf16 or fp32
  int out_fp32;
  float* lse;             // [B,Hq,N] or null
  int* status;
  const float* qscale;    // FP8 path only: per query row [B*Hq*N]
  const float* kscale;    // FP8 path only: per KV head [B*Hkv]
  const float* vscale;    // FP8 path with e4m3 P and V only: per KV head [B*Hkv]
};
// maps: [0] = Q (3D view [d, N, B*Hq], box 64 x 128), [1 + l] = K level l,
// [1 + L + l] = V level l (3D views [d, N/2^l, B*Hkv], box 64 x min(block/2^l, 64)).
cudaError_t launch_attention(const CUtensorMap* maps, const AttnArgs& a, int num_sms,
                             cudaStream_t s);
// The FP8 path (d = 128, bf16 output): Q and K maps over e4m3 codes, box
// 128 bytes wide (Q 128 rows, K levels min(block/2^l, 64) rows).  With pv,
// the V maps are over e4m3 codes too (same boxes as K) and P is e4m3.
cudaError_t launch_attention_fp8(const CUtensorMap* maps, const AttnArgs& a, bool pv, int num_sms, cudaStream_t s);

// ---- stage 3, backward ----------------------------------------------------
// D_i = dO_i . O_i and lse_i * log2(e) per query row, written into arrays
// padded to whole 128-row query tiles ([B*Hq][n_qtiles*128]); padding rows
// get lse2 = +inf (so their probabilities are exactly 0) and D = 0.
cudaError_t launch_bwd_prep(const void* out, const void* dout, const float* lse, float* lse2p, float* dp,
                            int64_t BHq, int N, int d, int n_qtiles, cudaStream_t s);

struct DqArgs {
  int B, Hq, Hkv, N, d, block, levels, causal;
  int n_items, n_qtiles;
  float scale_log2;       // sm_scale * log2(e)
  float sm_scale;
  const int* item_tile_off;
  const int* item_rows;
  const int* tile_seg_off;
  const int* segs;
  const int* queue;
  const float* lse2p;     // padded [B*Hq][n_qtiles*128]
  const float* dp;        // padded D
  void* dq;               // [B,Hq,N,d] bf16
  int* status;
};
// maps: [0] = Q, [1] = dO (3D [d, N, B*Hq], box 64 x 128), [2 + l] = K level l,
// [2 + L + l] = V level l (box 64 x min(block/2^l, 64)).
cudaError_t launch_dq(const CUtensorMap* maps, const DqArgs& a, int num_sms, cudaStream_t s);

// Transposed plan of the dK/dV kernel.  A work item is a 128-row tile of one
// pyramid level of one KV head: pooled rows [128 t, 128 t + 128) of level l,
// i.e. 128 / (block >> l) consecutive KV blocks.  Its entries are the query
// tiles (query head of the KV head's group, 128-row query tile) for which
// some block of the tile holds level l; each entry carries a bit mask, bit
// 2 jb + hf = block jb of the tile is at level l for query half hf (for
// 128-token blocks both half bits are equal).
struct TPlanArgs {
  int B, Hq, Hkv, N, block, nqb, nkb, levels, causal, n_qtiles;
  int n_items;
  int level_base[5];      // first item of level l; level_base[levels] = n_items
  int level_tiles[4];     // tiles per KV head at level l
  const uint8_t* mask;
  int* item_cnt;          // [n_items]
  int* item_off;          // [n_items + 1]
  int* entry_qt;          // [max entries]  h_local * n_qtiles + tq
  unsigned* entry_mask;   // [max entries]
};
cudaError_t launch_tplan(const TPlanArgs& a, cudaStream_t s);

struct DkvArgs {
  int B, Hq, Hkv, N, d, block, levels, causal, n_qtiles;
  int n_items;
  int level_base[5];
  int level_tiles[4];
  float scale_log2, sm_scale;
  const int* item_off;
  const int* entry_qt;
  const unsigned* entry_mask;
  const float* lse2p;
  const float* dp;
  float* dkl;             // fp32 level gradients, level l at dkl + level_off[l] (elements)
  float* dvl;
  int64_t level_off[4];   // element offset of level l ([B*Hkv][N >> l][d])
  int* status;
};
// maps: [0] = Q, [1] = dO (box 64 x 64 rows), [2 + l] = K level l, [2 + L + l] =
// V level l (box 64 x 128 rows).
cudaError_t launch_dkv(const CUtensorMap* maps, const DkvArgs& a, int num_sms, cudaStream_t s);

// dK[t] = dK^0[t] + sum_{l >= 1} dK^l[t >> l] / 2^l (same for V), fp32 level
// gradients -> bf16 output [B*Hkv][N][d].
cudaError_t launch_pool_bwd(const float* gl, const int64_t* level_off, void* out, int64_t BHkv, int N, int d,
                            int levels, cudaStream_t s);

// ---- FP8 operands -----------------------------------------------------------
// q [BHq][N][d] bf16 -> q8 codes (e4m3) and q_scale [BHq*N] (fp32, row max / 448);
// k (level 0) and the levels of k_pyr (element offsets level_off[l] of level l
// inside the pyramid buffer) -> k8 and k8_pyr codes at the same element
// offsets, and k_scale [BHkv] (fp32, head max of level 0 / 448).
// e4m3 codes of a per-head tensor and its pyramid levels ([BH][N >> l][d]
// bf16 each; level l > 0 at element offset level_off[l] of x_pyr / x8_pyr),
// one scale per head from level 0's largest magnitude: scale = max / 448.
cudaError_t launch_quantize_heads_fp8(const void* x, const void* x_pyr, const size_t* level_off, int64_t BH, int N,
                                     int d, int levels, uint8_t* x8, uint8_t* x8_pyr, float* scale, cudaStream_t s);
cudaError_t launch_quantize_qk_fp8(const void* q, const void* k, const void* k_pyr, const size_t* level_off,
                                   int64_t BHq, int64_t BHkv, int N, int d, int levels, uint8_t* q8, float* q_scale,
                                   uint8_t* k8, uint8_t* k8_pyr, float* k_scale, cudaStream_t s);

// Segment word of the tile plan: bits [0,2) level, [2,4) half mask (bit 0:
// query rows 0..63 of the tile use it, bit 1: rows 64..127; 0 marks a
// padding segment of zeros), [4,32) KV block index.
__host__ __device__ inline int seg_level(int w) { return w & 3; }
__host__ __device__ inline int seg_half(int w) { return (w >> 2) & 3; }
__host__ __device__ inline int seg_block(int w) { return w >> 4; }
__host__ __device__ inline int make_seg(int J, int l, int half) { return (J << 4) | (half << 2) | l; }

}  // namespace psa
