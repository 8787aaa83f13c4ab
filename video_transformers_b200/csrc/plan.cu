// plan.cu -- the tile planner of the PSA attention kernel: the decoupled
// block-tile layout (summary article "PSA: Pyramid Sparse Attention ...",
// Method: the logical block size is separated from the hardware tile size;
// news review, Methodology 5: blocks are grouped into tiles of a fixed
// compute budget).
//
// A work item is one 128-row query tile of one (b, h): query block I when
// block = 128, query blocks 2t and 2t+1 when block = 64.  Its KV side is the
// list of non-skipped (J, level) segments, each blk / 2^l pooled rows.  The
// planner orders the segments by level (so sizes descend through powers of
// two) and cuts the list into 128-row KV tiles; with that order no segment
// straddles a tile edge (or the 64-row half of a tile) and every segment
// starts on a multiple of its own size.  Only the last tile of an item can be
// partly empty; it is filled with padding segments that read zeros.
//
// plan_count (warp per item) -> plan_scan (one CTA) -> plan_fill (warp per
// item).  The queue is either head-major (items in their natural order, so
// the CTAs running at one time share one head's KV in L2) or sorted by tile
// count, largest first (the longest-processing-time order).
#include "internal.h"

namespace psa {
namespace {

struct ItemGeom {
  int b, h, tq, bh;
  int I0, I1;        // query blocks of half 0 / half 1 (I1 = -1 if none)
  int imax0, imax1;  // last query token of each half (-1 if the half is empty)
};

__device__ __forceinline__ ItemGeom item_geom(const PlanArgs& a, int item) {
  ItemGeom g;
  const int nqt = (a.N + 127) / 128;
  g.bh = item / nqt;
  g.tq = item - g.bh * nqt;
  g.b = g.bh / a.Hq;
  g.h = g.bh - g.b * a.Hq;
  if (a.block == 128) {
    g.I0 = g.tq;
    g.I1 = -1;
    g.imax0 = min(g.tq * 128 + 128, a.N) - 1;
    g.imax1 = -1;
  } else {
    g.I0 = 2 * g.tq;
    g.I1 = (2 * g.tq + 1 < a.nqb) ? 2 * g.tq + 1 : -1;
    g.imax0 = min(g.I0 * 64 + 64, a.N) - 1;
    g.imax1 = g.I1 >= 0 ? min(g.I1 * 64 + 64, a.N) - 1 : -1;
  }
  return g;
}

// Half mask of segment (J, l) for this item: bit h set iff query half h
// assigns level l to block J and at least one of its rows can see a token of
// the segment.
__device__ __forceinline__ int seg_halves(const PlanArgs& a, const ItemGeom& g, int J, int l) {
  const uint8_t* m = a.mask + static_cast<int64_t>(g.bh) * a.nqb * a.nkb;
  const int first_last_tok = J * a.block + (1 << l) - 1;   // last token of the segment's first pooled token
  int half = 0;
  if (m[static_cast<int64_t>(g.I0) * a.nkb + J] == l && (!a.causal || first_last_tok <= g.imax0)) half |= 1;
  if (a.block == 128) {
    half = half ? 3 : 0;
  } else if (g.I1 >= 0 && m[static_cast<int64_t>(g.I1) * a.nkb + J] == l &&
             (!a.causal || first_last_tok <= g.imax1)) {
    half |= 2;
  }
  return half;
}

// Padding of the last tile: from row `pos` up to the next multiple of 128,
// each pad as large as the alignment of its start allows (the lowest set bit
// of pos, at most 64), so every pad is aligned to its own size and none
// crosses a 64-row boundary.  pos is a multiple of the smallest segment, so
// every pad size is one of the available box sizes.
__device__ __forceinline__ int pad_size(int pos) {
  const int low = pos & -pos;
  return low < 64 ? low : 64;
}
__device__ __forceinline__ int pad_count(int pos) {
  int n = 0;
  while (pos & 127) { pos += pad_size(pos); ++n; }
  return n;
}
__device__ __forceinline__ int level_of_rows(int block, int rows) {
  int l = 0;
  while ((block >> l) > rows) ++l;
  return l;
}

__global__ void plan_count(const PlanArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= a.n_items) return;
  const ItemGeom g = item_geom(a, warp);
  int nseg = 0, rows = 0;
  for (int l = 0; l < a.levels; ++l) {
    int c = 0;
    for (int J = lane; J < a.nkb; J += 32) c += seg_halves(a, g, J, l) != 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    nseg += c;
    rows += c * (a.block >> l);
  }
  const int ntile = (rows + 127) / 128;
  const int npad = pad_count(rows);
  if (lane == 0) {
    a.item_nseg[warp] = nseg + npad;
    a.item_ntile[warp] = ntile;
    a.item_rows[warp] = rows;
  }
}

// single CTA: exclusive scans of segments and tiles, totals, queue histogram
__global__ void __launch_bounds__(1024) plan_scan(const PlanArgs a) {
  __shared__ long long wsum[3][32];
  __shared__ long long carry[3];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid < 3) carry[tid] = 0;
  for (int i = tid; i < a.n_hist; i += blockDim.x) a.hist[i] = 0;
  __syncthreads();
  for (int base = 0; base < a.n_items; base += blockDim.x) {
    const int i = base + tid;
    long long v[3] = {0, 0, 0};
    if (i < a.n_items) { v[0] = a.item_nseg[i]; v[1] = a.item_ntile[i]; v[2] = a.item_rows[i]; }
    long long inc[3] = {v[0], v[1], v[2]};
#pragma unroll
    for (int k = 0; k < 3; ++k) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, inc[k], o);
        if (lane >= o) inc[k] += y;
      }
      if (lane == 31) wsum[k][wid] = inc[k];
    }
    __syncthreads();
    long long off[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      long long w = 0;
      for (int x = 0; x < wid; ++x) w += wsum[k][x];
      off[k] = carry[k] + w + inc[k] - v[k];
    }
    if (i < a.n_items) {
      a.item_seg_off[i] = static_cast<int>(off[0]);
      a.item_tile_off[i] = static_cast<int>(off[1]);
      const int bin = min(static_cast<int>(v[1]), a.n_hist - 1);
      atomicAdd(&a.hist[bin], 1);
    }
    __syncthreads();
    if (tid == blockDim.x - 1) {
#pragma unroll
      for (int k = 0; k < 3; ++k) carry[k] = off[k] + v[k];
    }
    __syncthreads();
  }
  if (tid == 0) {
    a.item_seg_off[a.n_items] = static_cast<int>(carry[0]);
    a.item_tile_off[a.n_items] = static_cast<int>(carry[1]);
    a.tile_seg_off[carry[1]] = static_cast<int>(carry[0]);
    a.stats[0] = carry[1];
    a.stats[1] = carry[2];
    // queue start of each tile-count bin, largest counts first
    int acc = 0;
    for (int bin = a.n_hist - 1; bin >= 0; --bin) {
      const int c = a.hist[bin];
      a.hist[bin] = acc;
      acc += c;
    }
  }
}

__global__ void plan_fill(const PlanArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= a.n_items) return;
  const ItemGeom g = item_geom(a, warp);
  const int seg_base = a.item_seg_off[warp];
  const int tile_base = a.item_tile_off[warp];
  const int ntile = a.item_ntile[warp];
  int k = 0;      // segments written
  int row = 0;    // rows written
  for (int l = 0; l < a.levels; ++l) {
    const int sz = a.block >> l;
    for (int J0 = 0; J0 < a.nkb; J0 += 32) {
      const int J = J0 + lane;
      const int half = J < a.nkb ? seg_halves(a, g, J, l) : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, half != 0);
      if (half) {
        const int rank = __popc(bal & ((1u << lane) - 1u));
        const int idx = k + rank;
        const int r = row + rank * sz;
        a.segs[seg_base + idx] = make_seg(J, l, half);
        if ((r & 127) == 0) a.tile_seg_off[tile_base + (r >> 7)] = seg_base + idx;
      }
      const int n = __popc(bal);
      k += n;
      row += n * sz;
    }
  }
  if (lane == 0) {
    int pos = row;
    while (pos & 127) {
      const int sz = pad_size(pos);
      a.segs[seg_base + k] = make_seg(0, level_of_rows(a.block, sz), 0);
      ++k;
      pos += sz;
    }
    if (a.lpt_queue) {
      const int bin = min(ntile, a.n_hist - 1);
      const int pos = atomicAdd(&a.hist[bin], 1);
      a.queue[pos] = warp;
    } else {
      a.queue[warp] = warp;
    }
  }
}

}  // namespace

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s) {
  const int warps_per_cta = 8;
  const int grid = (a.n_items + warps_per_cta - 1) / warps_per_cta;
  plan_count<<<grid, 32 * warps_per_cta, 0, s>>>(a);
  plan_scan<<<1, 1024, 0, s>>>(a);
  plan_fill<<<grid, 32 * warps_per_cta, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace psa
