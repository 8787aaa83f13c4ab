// attn_common.cuh -- the record of one 64-row KV sub-tile shared by the
// attention kernels that walk the forward's tile plan (the forward kernel and
// the dQ kernel of the backward pass).  The producer warp writes it; the
// softmax warpgroup reads it to add the +ln 2^l bias (l in log2 units) of
// each column and to mask padding, ragged blocks, causal edges and, for
// 64-token blocks, the query half a segment does not serve.
#pragma once

#include <math_constants.h>

#include "internal.h"

namespace psa {

constexpr int kSubRows = 64;   // KV rows of a sub-tile

// The bias is kept per query half: with 64-token blocks a 128-row query tile
// holds two query blocks, and a segment may serve only one of them (its
// other half sees -inf).
struct alignas(16) SubInfo {
  float cb[2][4];            // level (or -inf) of each 16-column chunk, per query half (fast sub-tiles)
  int fast;                  // every chunk uniform per half, no padding, no ragged block, no causal edge
  int causal_check;          // slow sub-tiles: some column needs the causal test
  int pad[6];
  float bias[2][kSubRows];   // slow sub-tiles: level, or -inf, per query half
  int info[kSubRows];        // slow sub-tiles: last token each column covers (causal test)
};

// Writes the record of one sub-tile; called by all 32 lanes of the producer
// warp.  Lane s owns segment s of the current KV tile: `mine` = the segment
// has rows in this sub-tile, rows [lo, lo + cnt) of it land at sub-tile row
// `dst`; w = its segment word, l / half / J / rows its level, query-half
// mask, KV block and pooled rows; nseg segments in the tile; nl = N >> l;
// q0 = first query token of the item.
template <bool H2>
__device__ __forceinline__ void write_subinfo(SubInfo& ti, int lane, bool mine, int half, int l, int J, int rows,
                                              int lo, int cnt, int dst, int w, int nseg, int nl, int q0, int N,
                                              int block, int causal) {
  const int p_last = J * rows + lo + cnt;                // one past the last pooled row used here
  const int last_tok = (p_last << l) - 1;                // last token covered
  const bool seg_pad = mine && half == 0;
  const bool seg_ragged = mine && half != 0 && p_last > nl;
  const bool seg_causal = mine && half != 0 && causal && last_tok > q0;
  // an 8-row segment shares its 16-column chunk with the next one: the
  // chunk is uniform only if both serve the same query halves
  const int nxt_half = __shfl_down_sync(0xffffffffu, half, 1);
  const bool nxt_mine = __shfl_down_sync(0xffffffffu, mine ? 1 : 0, 1) != 0;
  const bool seg_split = H2 && mine && cnt < 16 && (dst & 15) == 0 &&
                         (!nxt_mine || lane + 1 >= nseg || nxt_half != half);
  const bool fast = !__any_sync(0xffffffffu, seg_pad || seg_ragged || seg_causal || seg_split);
  const bool causal_check = __any_sync(0xffffffffu, seg_causal);
  if (fast) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const unsigned bal = __ballot_sync(0xffffffffu, mine && dst <= 16 * k);
      const int src = bal ? 31 - __clz(bal) : 0;
      const int lev = __shfl_sync(0xffffffffu, l, src);
      const int hm = __shfl_sync(0xffffffffu, half, src);
      if (lane == k) ti.cb[0][k] = (hm & 1) ? static_cast<float>(lev) : -CUDART_INF_F;
      if (H2 && lane == 4 + k) ti.cb[1][k] = (hm & 2) ? static_cast<float>(lev) : -CUDART_INF_F;
    }
  } else {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int c = lane + 32 * m;
      float bias0 = -CUDART_INF_F, bias1 = -CUDART_INF_F;
      int inf = 0;
      for (int s = 0; s < nseg; ++s) {
        const int ms = __shfl_sync(0xffffffffu, mine ? 1 : 0, s);
        const int ds = __shfl_sync(0xffffffffu, dst, s);
        const int cs = __shfl_sync(0xffffffffu, cnt, s);
        const int los = __shfl_sync(0xffffffffu, lo, s);
        const int ws = __shfl_sync(0xffffffffu, w, s);
        if (ms && c >= ds && c < ds + cs) {
          const int ls = seg_level(ws), hf = seg_half(ws), Js = seg_block(ws);
          const int p = Js * (block >> ls) + los + (c - ds);
          const bool valid = hf != 0 && p < (N >> ls);
          bias0 = valid && (hf & 1) ? static_cast<float>(ls) : -CUDART_INF_F;
          bias1 = valid && (hf & 2) ? static_cast<float>(ls) : -CUDART_INF_F;
          inf = ((p + 1) << ls) - 1;
        }
      }
      ti.bias[0][c] = bias0;
      if (H2) ti.bias[1][c] = bias1;
      ti.info[c] = inf;
    }
  }
  if (lane == 0) { ti.fast = fast ? 1 : 0; ti.causal_check = causal_check ? 1 : 0; }
}

}  // namespace psa
