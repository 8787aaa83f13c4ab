// api.cu -- the C ABI of the PSA forward path (declared in include/psa.h):
// argument validation, workspace layout, TMA descriptor encoding and kernel
// launches.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"

namespace psa {

int device_sm_count() {
  constexpr int kDevs = 64;
  static std::atomic<int> cache[kDevs] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t set_smem_limit(const void* fn, int bytes) {
  struct Entry { const void* fn; int dev; int bytes; };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : done)
    if (x.fn == fn && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back({fn, dev, bytes});
  return e;
}

}  // namespace psa

namespace {

thread_local char g_err[512] = "";

psa_status_t fail(psa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

psa_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(PSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t elem_size(int dtype) { return dtype == PSA_DT_FP32 ? 4 : 2; }

// ------------------------------------------------------------------ driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Tensor map over `rank` dims (dims[0] innermost, contiguous), 128-byte
// swizzle, zero fill outside the tensor.
psa_status_t encode_map(CUtensorMap* m, CUtensorMapDataType type, const void* base, int rank, const uint64_t* dims,
                        const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(PSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; es[i] = 1; }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, type, rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PSA_OK;
}
psa_status_t encode_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                         const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

// [BH, rows, d] bf16 viewed as 3D {d, rows, BH}, box {64, box_rows, 1}
psa_status_t map3(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int d, int box_rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows), static_cast<uint64_t>(BH)};
  const uint64_t str[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(rows) * d * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(box_rows), 1};
  return encode_bf16(m, base, 3, dims, str, box);
}

// [BH, rows, d] e4m3 codes (one byte each) viewed as 3D {d, rows, BH}, box
// {d, box_rows, 1}; d = 128, so a box row is one 128-byte swizzle atom
psa_status_t map3_u8(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int d, int box_rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows), static_cast<uint64_t>(BH)};
  const uint64_t str[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows) * d};
  const uint32_t box[3] = {static_cast<uint32_t>(d), static_cast<uint32_t>(box_rows), 1};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 3, dims, str, box);
}

// [BH, N, d] bf16 viewed as 4D {d, step, N/step, BH}, box {64, 1, 128, 1}:
// one box row per `step` tokens starting at the chosen sub-row.
psa_status_t map4(CUtensorMap* m, const void* base, int64_t BH, int64_t N, int d, int step) {
  const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(step), static_cast<uint64_t>(N / step),
                            static_cast<uint64_t>(BH)};
  const uint64_t str[3] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(step) * d * 2,
                           static_cast<uint64_t>(N) * d * 2};
  const uint32_t box[4] = {64, 1, 128, 1};
  return encode_bf16(m, base, 4, dims, str, box);
}

int num_sms() { return psa::device_sm_count(); }

// ------------------------------------------------------------------ validation
psa_status_t check_shape(const psa_shape_t* s) {
  if (!s) return fail(PSA_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->N < 1 || s->d < 1 || s->block < 1 || s->levels < 1)
    return fail(PSA_ERR_INVALID_ARG, "shape fields must be positive");
  if (s->dtype != PSA_DT_BF16 && s->dtype != PSA_DT_FP32) return fail(PSA_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
  if (s->d != 64 && s->d != 128) return fail(PSA_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", s->d);
  if (s->block != 64 && s->block != 128) return fail(PSA_ERR_UNSUPPORTED, "block %d not in {64, 128}", s->block);
  if (s->levels > PSA_MAX_LEVELS) return fail(PSA_ERR_UNSUPPORTED, "levels %d > %d", s->levels, PSA_MAX_LEVELS);
  const int g = 1 << (s->levels - 1);
  if (s->block % g || s->N % g) return fail(PSA_ERR_UNSUPPORTED, "block and N must be multiples of 2^(L-1) = %d", g);
  if (s->Hq % s->Hkv) return fail(PSA_ERR_UNSUPPORTED, "Hq %d not a multiple of Hkv %d", s->Hq, s->Hkv);
  if (static_cast<int64_t>(s->B) * s->Hq * s->N * s->d >= (1ll << 31))
    return fail(PSA_ERR_UNSUPPORTED, "B*Hq*N*d must be < 2^31");
  if (ceil_div(s->N, s->block) > PSA_MAX_KV_BLOCKS) return fail(PSA_ERR_UNSUPPORTED, "more than %d KV blocks", PSA_MAX_KV_BLOCKS);
  return PSA_OK;
}

psa_status_t check_ptr(const void* p, const char* name, bool required = true) {
  if (!p) return required ? fail(PSA_ERR_INVALID_ARG, "%s is NULL", name) : PSA_OK;
  if (!aligned16(p)) return fail(PSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return PSA_OK;
}

#define PSA_TRY(x)                      \
  do {                                  \
    psa_status_t st__ = (x);            \
    if (st__ != PSA_OK) return st__;    \
  } while (0)
#define PSA_CUDA(x, what)                              \
  do {                                                 \
    cudaError_t e__ = (x);                             \
    if (e__ != cudaSuccess) return cuda_fail(e__, what); \
  } while (0)

// ------------------------------------------------------------------ pyramid layout
size_t level_rows_total(const psa_shape_t* s, int upto) {   // sum over l in [1, upto) of N/2^l
  size_t r = 0;
  for (int l = 1; l < upto; ++l) r += static_cast<size_t>(s->N >> l);
  return r;
}
size_t pyr_level_offset(const psa_shape_t* s, int level, size_t esize) {
  return static_cast<size_t>(s->B) * s->Hkv * level_rows_total(s, level) * s->d * esize;
}
size_t pyr_bytes(const psa_shape_t* s, size_t esize) { return pyr_level_offset(s, s->levels, esize); }

// ------------------------------------------------------------------ mask workspace
struct MaskLayout {
  size_t status, blocklse, rowlse, q16, k16, qmean, kmean, total;
  int rows, step, rpb, cols, cpb;
};
MaskLayout mask_layout(const psa_shape_t* s, const psa_mask_params_t* p) {
  MaskLayout L{};
  const int nqb = static_cast<int>(ceil_div(s->N, s->block));
  const int nkb = nqb;
  if (p->mode == PSA_MASK_SAMPLE) {
    L.step = s->block / 8;
    L.rpb = 8;
    L.rows = nqb * 8;
    L.cols = s->N;
    L.cpb = s->block;
  } else if (p->mode == PSA_MASK_MEANKEY) {
    L.step = s->block;
    L.rpb = 1;
    L.rows = nqb;
    L.cols = nkb;
    L.cpb = 1;
  } else {
    L.step = p->stride;
    L.rpb = s->block / p->stride;
    L.rows = s->N / p->stride;
    L.cols = s->N / p->stride;
    L.cpb = s->block / p->stride;
  }
  const size_t BHq = static_cast<size_t>(s->B) * s->Hq;
  size_t off = 256;
  L.status = 0;
  L.blocklse = off; off = align_up(off + BHq * nkb * L.rows * 4, 256);
  L.rowlse = off;   off = align_up(off + psa::kScore2Parts * BHq * L.rows * 4, 256);   // row-LSE partials
  if (p->mode == PSA_MASK_MEANKEY) {
    // block means in fp64; the mean-key scorer reads the inputs directly
    L.qmean = off; off = align_up(off + BHq * nqb * s->d * 8, 256);
    L.kmean = off; off = align_up(off + static_cast<size_t>(s->B) * s->Hkv * nkb * s->d * 8, 256);
  } else if (s->dtype == PSA_DT_FP32) {
    L.q16 = off; off = align_up(off + BHq * s->N * s->d * 2, 256);
    L.k16 = off; off = align_up(off + static_cast<size_t>(s->B) * s->Hkv * s->N * s->d * 2, 256);
  }
  L.total = off;
  return L;
}

psa_status_t check_mask_params(const psa_shape_t* s, const psa_mask_params_t* p) {
  if (!p) return fail(PSA_ERR_INVALID_ARG, "params is NULL");
  if (p->mode != PSA_MASK_SAMPLE && p->mode != PSA_MASK_ANTIDIAG && p->mode != PSA_MASK_MEANKEY)
    return fail(PSA_ERR_INVALID_ARG, "unknown mask mode %d", p->mode);
  if (p->policy != PSA_POLICY_MASS && p->policy != PSA_POLICY_QUANTILE)
    return fail(PSA_ERR_INVALID_ARG, "unknown level policy %d", p->policy);
  if (p->n_thresholds != s->levels) return fail(PSA_ERR_INVALID_ARG, "n_thresholds %d != levels %d", p->n_thresholds, s->levels);
  for (int i = 0; i < p->n_thresholds; ++i)
    if (!(p->thresholds[i] == p->thresholds[i])) return fail(PSA_ERR_INVALID_ARG, "threshold %d is NaN", i);
  if (!(p->sm_scale > 0.f) || p->sm_scale != p->sm_scale) return fail(PSA_ERR_INVALID_ARG, "sm_scale must be > 0");
  if (p->n_dense_prefix < 0) return fail(PSA_ERR_INVALID_ARG, "n_dense_prefix < 0");
  if (p->mode == PSA_MASK_SAMPLE) {
    if (p->n_samples != 8) return fail(PSA_ERR_UNSUPPORTED, "n_samples must be 8");
    if (s->N % (s->block / 8)) return fail(PSA_ERR_UNSUPPORTED, "sampling needs N %% (block/8) == 0");
  } else if (p->mode == PSA_MASK_MEANKEY) {
    // no alignment needed: the block means read every token once
  } else {
    const int S = p->stride;
    if (S != 1 && S != 2 && S != 4 && S != 8 && S != 16) return fail(PSA_ERR_UNSUPPORTED, "stride %d not in {1,2,4,8,16}", S);
    if (s->N % S) return fail(PSA_ERR_UNSUPPORTED, "antidiagonal scoring needs N %% stride == 0");
    if (s->block / S < 8) return fail(PSA_ERR_UNSUPPORTED, "block / stride must be >= 8");
  }
  return PSA_OK;
}

// ------------------------------------------------------------------ attention workspace
struct AttnLayout {
  size_t status, stats, nseg, ntile, nrows, seg_off, tile_off, hist, queue, tile_seg_off, segs;
  size_t q16, k16, v16, kp16, vp16, total;
  int n_items, n_qtiles, n_hist;
  int64_t max_tiles, max_segs;
};
AttnLayout attn_layout(const psa_shape_t* s) {
  AttnLayout L{};
  const int nkb = static_cast<int>(ceil_div(s->N, s->block));
  L.n_qtiles = static_cast<int>(ceil_div(s->N, 128));
  L.n_items = s->B * s->Hq * L.n_qtiles;
  L.n_hist = nkb + 2;
  L.max_tiles = static_cast<int64_t>(L.n_items) * nkb;
  const int per_level = s->block == 64 ? 2 * nkb : nkb;
  L.max_segs = static_cast<int64_t>(L.n_items) * (per_level + s->levels);
  const size_t n = static_cast<size_t>(L.n_items);
  size_t off = 0;
  L.status = off; L.stats = 64; off = 256;   // [0, 36): status word + time-out record
  L.nseg = off;     off = align_up(off + n * 4, 256);
  L.ntile = off;    off = align_up(off + n * 4, 256);
  L.nrows = off;    off = align_up(off + n * 4, 256);
  L.seg_off = off;  off = align_up(off + (n + 1) * 4, 256);
  L.tile_off = off; off = align_up(off + (n + 1) * 4, 256);
  L.hist = off;     off = align_up(off + static_cast<size_t>(L.n_hist) * 4, 256);
  L.queue = off;    off = align_up(off + n * 4, 256);
  L.tile_seg_off = off; off = align_up(off + static_cast<size_t>(L.max_tiles + 1) * 4, 256);
  L.segs = off;     off = align_up(off + static_cast<size_t>(L.max_segs) * 4, 256);
  if (s->dtype == PSA_DT_FP32) {
    const size_t qn = static_cast<size_t>(s->B) * s->Hq * s->N * s->d;
    const size_t kn = static_cast<size_t>(s->B) * s->Hkv * s->N * s->d;
    L.q16 = off;  off = align_up(off + qn * 2, 256);
    L.k16 = off;  off = align_up(off + kn * 2, 256);
    L.v16 = off;  off = align_up(off + kn * 2, 256);
    L.kp16 = off; off = align_up(off + pyr_bytes(s, 2), 256);
    L.vp16 = off; off = align_up(off + pyr_bytes(s, 2), 256);
  }
  L.total = off;
  return L;
}

// Byte offset, inside every workspace header, of the debug words read by the
// attention kernel: the 64-bit limit of its debug trap wait (0 = the
// built-in limit) at 40, the trap flag at 48.
constexpr size_t kWaitLimitOffset = 40;

// Reads the status word and time-out record at the start of a workspace
// header, clears them (36 bytes: the debug words after them are kept), and
// turns them into a status and message.
psa_status_t read_status(void* hdr, void* stream) {
  int w[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  cudaStream_t str = static_cast<cudaStream_t>(stream);
  PSA_CUDA(cudaMemcpyAsync(w, hdr, sizeof(w), cudaMemcpyDeviceToHost, str), "status copy");
  PSA_CUDA(cudaMemsetAsync(hdr, 0, sizeof(w), str), "status clear");
  PSA_CUDA(cudaStreamSynchronize(str), "status sync");
  if (w[0] == 0) return PSA_OK;
  return fail(static_cast<psa_status_t>(w[0]),
              "device status %d: a bounded wait ran out (site %d, block %d, thread %d, counters %d %d %d %d)",
              w[0], w[2], w[3], w[4], w[5], w[6], w[7], w[8]);
}

// ------------------------------------------------------------------ backward workspace
struct BwdLayout {
  AttnLayout fwd;                  // the forward's tile plan, at the start of the workspace
  size_t lse2p, dp, tcnt, toff, eqt, emask, dkl, dvl, total;
  int n_titems, level_base[5], level_tiles[4];
  int64_t max_entries, level_off[4];
};
BwdLayout bwd_layout(const psa_shape_t* s) {
  BwdLayout L{};
  L.fwd = attn_layout(s);
  size_t off = L.fwd.total;
  const size_t BHq = static_cast<size_t>(s->B) * s->Hq;
  const int64_t BHkv = static_cast<int64_t>(s->B) * s->Hkv;
  const size_t padded = BHq * static_cast<size_t>(L.fwd.n_qtiles) * 128;
  L.lse2p = off; off = align_up(off + padded * 4, 256);
  L.dp = off;    off = align_up(off + padded * 4, 256);
  int n = 0;
  int64_t elems = 0;
  for (int l = 0; l < s->levels; ++l) {
    L.level_base[l] = n;
    L.level_tiles[l] = static_cast<int>(ceil_div(s->N >> l, 128));
    n += static_cast<int>(BHkv * L.level_tiles[l]);
    L.level_off[l] = elems;
    elems += BHkv * (s->N >> l) * s->d;
  }
  for (int l = s->levels; l < 4; ++l) { L.level_tiles[l] = 0; L.level_off[l] = 0; }
  L.level_base[s->levels] = n;
  L.n_titems = n;
  L.max_entries = static_cast<int64_t>(n) * (s->Hq / s->Hkv) * L.fwd.n_qtiles;
  L.tcnt = off;  off = align_up(off + static_cast<size_t>(n) * 4, 256);
  L.toff = off;  off = align_up(off + static_cast<size_t>(n + 1) * 4, 256);
  L.eqt = off;   off = align_up(off + static_cast<size_t>(L.max_entries) * 4, 256);
  L.emask = off; off = align_up(off + static_cast<size_t>(L.max_entries) * 4, 256);
  L.dkl = off;   off = align_up(off + static_cast<size_t>(elems) * 4, 256);
  L.dvl = off;   off = align_up(off + static_cast<size_t>(elems) * 4, 256);
  L.total = off;
  return L;
}

// ------------------------------------------------------------------ FP8 workspace
struct Fp8Layout {
  AttnLayout fwd;                  // the tile plan, at the start of the workspace
  size_t q8, qs, k8, kp8, ks, v8, vp8, vs, total;
};
Fp8Layout fp8_layout(const psa_shape_t* s) {
  Fp8Layout L{};
  L.fwd = attn_layout(s);
  size_t off = L.fwd.total;
  const size_t BHq = static_cast<size_t>(s->B) * s->Hq, BHkv = static_cast<size_t>(s->B) * s->Hkv;
  L.q8 = off;  off = align_up(off + BHq * s->N * s->d, 256);
  L.qs = off;  off = align_up(off + BHq * s->N * 4, 256);
  L.k8 = off;  off = align_up(off + BHkv * s->N * s->d, 256);
  L.kp8 = off; off = align_up(off + pyr_bytes(s, 1), 256);
  L.ks = off;  off = align_up(off + BHkv * 4, 256);
  L.v8 = off;  off = align_up(off + BHkv * s->N * s->d, 256);      // e4m3 values (the P.V path only)
  L.vp8 = off; off = align_up(off + pyr_bytes(s, 1), 256);
  L.vs = off;  off = align_up(off + BHkv * 4, 256);
  L.total = off;
  return L;
}

psa_status_t check_fp8_shape(const psa_shape_t* s) {
  PSA_TRY(check_shape(s));
  if (s->dtype != PSA_DT_BF16) return fail(PSA_ERR_UNSUPPORTED, "the FP8 path takes bf16 tensors");
  if (s->d != 128) return fail(PSA_ERR_UNSUPPORTED, "the FP8 path is built for head dim 128");
  return PSA_OK;
}

psa_status_t attention_fp8(const psa_shape_t* s, const void* q, const void* k, const void* v, const void* k_pyr,
                           const void* v_pyr, const uint8_t* mask, float sm_scale, void* out, float* lse, void* ws,
                           size_t ws_bytes, void* stream, bool pv) {
  g_err[0] = 0;
  PSA_TRY(check_fp8_shape(s));
  PSA_TRY(check_ptr(q, "q"));
  PSA_TRY(check_ptr(k, "k"));
  PSA_TRY(check_ptr(v, "v"));
  PSA_TRY(check_ptr(out, "out"));
  if (s->levels > 1) {
    PSA_TRY(check_ptr(k_pyr, "k_pyr"));
    PSA_TRY(check_ptr(v_pyr, "v_pyr"));
  }
  if (!mask) return fail(PSA_ERR_INVALID_ARG, "mask is NULL");
  PSA_TRY(check_ptr(lse, "lse", false));
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return fail(PSA_ERR_INVALID_ARG, "sm_scale must be > 0");
  const Fp8Layout L = fp8_layout(s);
  if (L.fwd.max_segs >= (1ll << 31) || L.fwd.max_tiles >= (1ll << 31))
    return fail(PSA_ERR_UNSUPPORTED, "tile plan would exceed 2^31 entries");
  if (!ws || !aligned16(ws)) return fail(PSA_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
  if (ws_bytes < L.total) return fail(PSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const int64_t BHq = static_cast<int64_t>(s->B) * s->Hq, BHkv = static_cast<int64_t>(s->B) * s->Hkv;
  uint8_t* q8 = reinterpret_cast<uint8_t*>(w + L.q8);
  uint8_t* k8 = reinterpret_cast<uint8_t*>(w + L.k8);
  uint8_t* kp8 = reinterpret_cast<uint8_t*>(w + L.kp8);
  float* qs = reinterpret_cast<float*>(w + L.qs);
  float* ks = reinterpret_cast<float*>(w + L.ks);
  size_t off[PSA_MAX_LEVELS] = {0, 0, 0, 0};
  for (int l = 1; l < s->levels; ++l) off[l] = pyr_level_offset(s, l, 1);
  PSA_CUDA(psa::launch_quantize_qk_fp8(q, k, k_pyr, off, BHq, BHkv, s->N, s->d, s->levels, q8, qs, k8, kp8, ks, st),
           "fp8 quantize launch");
  uint8_t* v8 = reinterpret_cast<uint8_t*>(w + L.v8);
  uint8_t* vp8 = reinterpret_cast<uint8_t*>(w + L.vp8);
  float* vs = reinterpret_cast<float*>(w + L.vs);
  if (pv)
    PSA_CUDA(psa::launch_quantize_heads_fp8(v, v_pyr, off, BHkv, s->N, s->d, s->levels, v8, vp8, vs, st),
             "fp8 value quantize launch");
  CUtensorMap maps[9];
  PSA_TRY(map3_u8(&maps[0], q8, BHq, s->N, s->d, 128));
  const char* vp = static_cast<const char*>(v_pyr);
  for (int l = 0; l < s->levels; ++l) {
    const void* kb = l == 0 ? static_cast<const void*>(k8) : static_cast<const void*>(kp8 + off[l]);
    const void* vb = l == 0 ? v : static_cast<const void*>(vp + pyr_level_offset(s, l, 2));
    const int box = (s->block >> l) < 64 ? (s->block >> l) : 64;
    PSA_TRY(map3_u8(&maps[1 + l], kb, BHkv, s->N >> l, s->d, box));
    if (pv) {
      const void* vb8 = l == 0 ? static_cast<const void*>(v8) : static_cast<const void*>(vp8 + off[l]);
      PSA_TRY(map3_u8(&maps[1 + s->levels + l], vb8, BHkv, s->N >> l, s->d, box));
    } else {
      PSA_TRY(map3(&maps[1 + s->levels + l], vb, BHkv, s->N >> l, s->d, box));
    }
  }
  const int nkb = static_cast<int>(ceil_div(s->N, s->block));
  psa::PlanArgs pa{};
  pa.B = s->B; pa.Hq = s->Hq; pa.N = s->N; pa.block = s->block; pa.nqb = nkb; pa.nkb = nkb;
  pa.levels = s->levels; pa.causal = s->causal != 0; pa.n_items = L.fwd.n_items; pa.mask = mask;
  pa.item_nseg = reinterpret_cast<int*>(w + L.fwd.nseg);
  pa.item_ntile = reinterpret_cast<int*>(w + L.fwd.ntile);
  pa.item_rows = reinterpret_cast<int*>(w + L.fwd.nrows);
  pa.item_seg_off = reinterpret_cast<int*>(w + L.fwd.seg_off);
  pa.item_tile_off = reinterpret_cast<int*>(w + L.fwd.tile_off);
  pa.tile_seg_off = reinterpret_cast<int*>(w + L.fwd.tile_seg_off);
  pa.segs = reinterpret_cast<int*>(w + L.fwd.segs);
  pa.queue = reinterpret_cast<int*>(w + L.fwd.queue);
  pa.hist = reinterpret_cast<int*>(w + L.fwd.hist);
  pa.n_hist = L.fwd.n_hist;
  pa.lpt_queue = 0;
  pa.stats = reinterpret_cast<long long*>(w + L.fwd.stats);
  PSA_CUDA(psa::launch_plan(pa, st), "plan launch");
  psa::AttnArgs aa{};
  aa.B = s->B; aa.Hq = s->Hq; aa.Hkv = s->Hkv; aa.N = s->N; aa.d = s->d; aa.block = s->block;
  aa.levels = s->levels; aa.causal = s->causal != 0; aa.n_items = L.fwd.n_items; aa.n_qtiles = L.fwd.n_qtiles;
  aa.scale_log2 = sm_scale * 1.4426950408889634f;
  aa.item_tile_off = pa.item_tile_off;
  aa.item_rows = pa.item_rows;
  aa.tile_seg_off = pa.tile_seg_off;
  aa.segs = pa.segs;
  aa.queue = pa.queue;
  aa.out = out;
  aa.out_fp32 = 0;
  aa.lse = lse;
  aa.status = reinterpret_cast<int*>(w + L.fwd.status);
  aa.qscale = qs;
  aa.kscale = ks;
  aa.vscale = pv ? vs : nullptr;
  PSA_CUDA(psa::launch_attention_fp8(maps, aa, pv, num_sms(), st), "fp8 attention launch");
  return PSA_OK;
}

}  // namespace

extern "C" {

const char* psa_last_error(void) { return g_err; }
int32_t psa_version(void) { return 100; }

size_t psa_pyramid_bytes(const psa_shape_t* s) {
  if (check_shape(s) != PSA_OK) return 0;
  return pyr_bytes(s, elem_size(s->dtype));
}

size_t psa_pyramid_level_offset(const psa_shape_t* s, int level) {
  if (check_shape(s) != PSA_OK || level < 1 || level >= s->levels) return 0;
  return pyr_level_offset(s, level, elem_size(s->dtype));
}

psa_status_t psa_build_pyramid(const psa_shape_t* s, const void* k, const void* v, void* k_pyr, void* v_pyr,
                               float* blockcos, void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  PSA_TRY(check_ptr(k, "k"));
  PSA_TRY(check_ptr(v, "v"));
  if (s->levels > 1) {
    PSA_TRY(check_ptr(k_pyr, "k_pyr"));
    PSA_TRY(check_ptr(v_pyr, "v_pyr"));
  }
  PSA_TRY(check_ptr(blockcos, "blockcos", false));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t es = elem_size(s->dtype);
  size_t off[PSA_MAX_LEVELS] = {0, 0, 0, 0};
  for (int l = 1; l < s->levels; ++l) off[l] = pyr_level_offset(s, l, es);
  const int64_t BH = static_cast<int64_t>(s->B) * s->Hkv;
  PSA_CUDA(psa::launch_pyramid(k, v, k_pyr, v_pyr, BH, s->N, s->d, s->levels, static_cast<int>(es), off, st),
           "pyramid launch");
  if (blockcos) PSA_CUDA(psa::launch_blockcos(k, blockcos, BH, s->N, s->d, s->block, static_cast<int>(es), st), "blockcos launch");
  return PSA_OK;
}

size_t psa_mask_workspace_bytes(const psa_shape_t* s, const psa_mask_params_t* p) {
  if (check_shape(s) != PSA_OK || check_mask_params(s, p) != PSA_OK) return 0;
  return mask_layout(s, p).total;
}

psa_status_t psa_make_mask(const psa_shape_t* s, const psa_mask_params_t* p, const void* q, const void* k,
                           const float* blockcos, uint8_t* mask, float* mass_out, void* ws, size_t ws_bytes,
                           void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  PSA_TRY(check_mask_params(s, p));
  PSA_TRY(check_ptr(q, "q"));
  PSA_TRY(check_ptr(k, "k"));
  if (!mask) return fail(PSA_ERR_INVALID_ARG, "mask is NULL");
  PSA_TRY(check_ptr(mass_out, "mass_out", false));
  if (p->cos_min > -2.f) PSA_TRY(check_ptr(blockcos, "blockcos (required when cos_min > -2)"));
  const MaskLayout L = mask_layout(s, p);
  if (!ws || !aligned16(ws)) return fail(PSA_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
  if (ws_bytes < L.total) return fail(PSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const int64_t BHq = static_cast<int64_t>(s->B) * s->Hq, BHkv = static_cast<int64_t>(s->B) * s->Hkv;
  const int nkb = static_cast<int>(ceil_div(s->N, s->block));
  psa::SelectArgs se{};
  se.B = s->B; se.Hq = s->Hq; se.Hkv = s->Hkv; se.N = s->N; se.block = s->block;
  se.nqb = nkb; se.nkb = nkb; se.levels = s->levels; se.causal = s->causal != 0;
  se.mode = p->mode; se.rows = L.rows; se.rows_per_block = L.rpb; se.step = L.step;
  se.policy = p->policy;
  for (int i = 0; i < 8; ++i) se.thresholds[i] = i < p->n_thresholds ? p->thresholds[i] : 3.0e38f;
  se.cos_min = p->cos_min;
  se.n_dense_prefix = p->n_dense_prefix;
  se.blockcos = p->cos_min > -2.f ? blockcos : nullptr;
  se.mask = mask;
  se.mass_out = mass_out;
  se.blocklse = reinterpret_cast<float*>(w + L.blocklse);
  se.rowlse = reinterpret_cast<float*>(w + L.rowlse);
  // partials per row: one per column part of the paired sampling score,
  // else two (the one-row-tile score's warpgroups; the mean-key scorer)
  se.n_part = (p->mode == PSA_MASK_SAMPLE && s->d == 128) ? psa::kScore2Parts : 2;
  if (p->mode == PSA_MASK_MEANKEY) {
    const int es = static_cast<int>(elem_size(s->dtype));
    double* qm = reinterpret_cast<double*>(w + L.qmean);
    double* km = reinterpret_cast<double*>(w + L.kmean);
    PSA_CUDA(psa::launch_blockmean(q, qm, BHq, s->N, s->d, s->block, es, true, st), "query block means");
    PSA_CUDA(psa::launch_blockmean(k, km, BHkv, s->N, s->d, s->block, es, true, st), "key block means");
    psa::MeanKeyArgs ma{};
    ma.BHq = static_cast<int>(BHq); ma.Hq = s->Hq; ma.Hkv = s->Hkv; ma.d = s->d;
    ma.nqb = nkb; ma.nkb = nkb; ma.causal = s->causal != 0;
    ma.scale_log2 = static_cast<double>(p->sm_scale) * 1.4426950408889634;
    ma.qmean = qm; ma.kmeanT = km;
    ma.blocklse = reinterpret_cast<float*>(w + L.blocklse);
    ma.rowlse = reinterpret_cast<float*>(w + L.rowlse);
    PSA_CUDA(psa::launch_meankey_score(ma, st), "mean-key score launch");
    se.S = 1;
    PSA_CUDA(psa::launch_select(se, st), "select launch");
    return PSA_OK;
  }
  const void* q16 = q;
  const void* k16 = k;
  if (s->dtype == PSA_DT_FP32) {
    PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(q), w + L.q16, BHq * s->N * s->d, st), "cast q");
    PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(k), w + L.k16, BHkv * s->N * s->d, st), "cast k");
    q16 = w + L.q16;
    k16 = w + L.k16;
  }
  CUtensorMap mA, mB;
  PSA_TRY(map4(&mA, q16, BHq, s->N, s->d, L.step));
  PSA_TRY(map4(&mB, k16, BHkv, s->N, s->d, p->mode == PSA_MASK_SAMPLE ? 1 : p->stride));
  psa::ScoreArgs sa{};
  sa.BHq = static_cast<int>(BHq); sa.Hq = s->Hq; sa.Hkv = s->Hkv; sa.N = s->N; sa.d = s->d;
  sa.block = s->block; sa.nkb = nkb; sa.mode = p->mode; sa.step = L.step;
  sa.S = p->mode == PSA_MASK_SAMPLE ? 1 : p->stride;
  sa.rows = L.rows; sa.cols = L.cols; sa.rows_per_block = L.rpb; sa.cols_per_block = L.cpb;
  sa.causal = s->causal != 0;
  const float sc = p->mode == PSA_MASK_SAMPLE ? p->sm_scale : p->sm_scale / static_cast<float>(p->stride);
  sa.scale_log2 = sc * 1.4426950408889634f;
  sa.blocklse = reinterpret_cast<float*>(w + L.blocklse);
  sa.rowlse = reinterpret_cast<float*>(w + L.rowlse);
  sa.status = reinterpret_cast<int*>(w + L.status);
  PSA_CUDA(psa::launch_score(&mA, &mB, sa, num_sms(), st), "score launch");
  se.S = sa.S;
  PSA_CUDA(psa::launch_select(se, st), "select launch");
  return PSA_OK;
}

size_t psa_attention_workspace_bytes(const psa_shape_t* s) {
  if (check_shape(s) != PSA_OK) return 0;
  return attn_layout(s).total;
}

psa_status_t psa_attention_fwd(const psa_shape_t* s, const void* q, const void* k, const void* v, const void* k_pyr,
                               const void* v_pyr, const uint8_t* mask, float sm_scale, void* out, float* lse,
                               void* ws, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  PSA_TRY(check_ptr(q, "q"));
  PSA_TRY(check_ptr(k, "k"));
  PSA_TRY(check_ptr(v, "v"));
  PSA_TRY(check_ptr(out, "out"));
  if (s->levels > 1) {
    PSA_TRY(check_ptr(k_pyr, "k_pyr"));
    PSA_TRY(check_ptr(v_pyr, "v_pyr"));
  }
  if (!mask) return fail(PSA_ERR_INVALID_ARG, "mask is NULL");
  PSA_TRY(check_ptr(lse, "lse", false));
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return fail(PSA_ERR_INVALID_ARG, "sm_scale must be > 0");
  const AttnLayout L = attn_layout(s);
  if (L.max_segs >= (1ll << 31) || L.max_tiles >= (1ll << 31))
    return fail(PSA_ERR_UNSUPPORTED, "tile plan would exceed 2^31 entries");
  if (!ws || !aligned16(ws)) return fail(PSA_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
  if (ws_bytes < L.total) return fail(PSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const int64_t BHq = static_cast<int64_t>(s->B) * s->Hq, BHkv = static_cast<int64_t>(s->B) * s->Hkv;
  const void* q16 = q;
  const void* k16 = k;
  const void* v16 = v;
  const char* kp16 = static_cast<const char*>(k_pyr);
  const char* vp16 = static_cast<const char*>(v_pyr);
  if (s->dtype == PSA_DT_FP32) {
    PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(q), w + L.q16, BHq * s->N * s->d, st), "cast q");
    PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(k), w + L.k16, BHkv * s->N * s->d, st), "cast k");
    PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(v), w + L.v16, BHkv * s->N * s->d, st), "cast v");
    const int64_t pn = static_cast<int64_t>(pyr_bytes(s, 4) / 4);
    if (pn > 0) {
      PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(k_pyr), w + L.kp16, pn, st), "cast k_pyr");
      PSA_CUDA(psa::launch_cast_bf16(static_cast<const float*>(v_pyr), w + L.vp16, pn, st), "cast v_pyr");
    }
    q16 = w + L.q16; k16 = w + L.k16; v16 = w + L.v16;
    kp16 = w + L.kp16; vp16 = w + L.vp16;
  }
  CUtensorMap maps[9];
  PSA_TRY(map3(&maps[0], q16, BHq, s->N, s->d, 128));
  for (int l = 0; l < s->levels; ++l) {
    const void* kb = l == 0 ? k16 : static_cast<const void*>(kp16 + pyr_level_offset(s, l, 2));
    const void* vb = l == 0 ? v16 : static_cast<const void*>(vp16 + pyr_level_offset(s, l, 2));
    const int box = (s->block >> l) < 64 ? (s->block >> l) : 64;   // KV sub-tiles are 64 rows
    PSA_TRY(map3(&maps[1 + l], kb, BHkv, s->N >> l, s->d, box));
    PSA_TRY(map3(&maps[1 + s->levels + l], vb, BHkv, s->N >> l, s->d, box));
  }
  const int nkb = static_cast<int>(ceil_div(s->N, s->block));
  psa::PlanArgs pa{};
  pa.B = s->B; pa.Hq = s->Hq; pa.N = s->N; pa.block = s->block; pa.nqb = nkb; pa.nkb = nkb;
  pa.levels = s->levels; pa.causal = s->causal != 0; pa.n_items = L.n_items; pa.mask = mask;
  pa.item_nseg = reinterpret_cast<int*>(w + L.nseg);
  pa.item_ntile = reinterpret_cast<int*>(w + L.ntile);
  pa.item_rows = reinterpret_cast<int*>(w + L.nrows);
  pa.item_seg_off = reinterpret_cast<int*>(w + L.seg_off);
  pa.item_tile_off = reinterpret_cast<int*>(w + L.tile_off);
  pa.tile_seg_off = reinterpret_cast<int*>(w + L.tile_seg_off);
  pa.segs = reinterpret_cast<int*>(w + L.segs);
  pa.queue = reinterpret_cast<int*>(w + L.queue);
  pa.hist = reinterpret_cast<int*>(w + L.hist);
  pa.n_hist = L.n_hist;
  pa.lpt_queue = 0;
  pa.stats = reinterpret_cast<long long*>(w + L.stats);
  PSA_CUDA(psa::launch_plan(pa, st), "plan launch");

  psa::AttnArgs aa{};
  aa.B = s->B; aa.Hq = s->Hq; aa.Hkv = s->Hkv; aa.N = s->N; aa.d = s->d; aa.block = s->block;
  aa.levels = s->levels; aa.causal = s->causal != 0; aa.n_items = L.n_items; aa.n_qtiles = L.n_qtiles;
  aa.scale_log2 = sm_scale * 1.4426950408889634f;
  aa.item_tile_off = pa.item_tile_off;
  aa.item_rows = pa.item_rows;
  aa.tile_seg_off = pa.tile_seg_off;
  aa.segs = pa.segs;
  aa.queue = pa.queue;
  aa.out = out;
  aa.out_fp32 = s->dtype == PSA_DT_FP32;
  aa.lse = lse;
  aa.status = reinterpret_cast<int*>(w + L.status);
  PSA_CUDA(psa::launch_attention(maps, aa, num_sms(), st), "attention launch");
  return PSA_OK;
}

size_t psa_attention_bwd_workspace_bytes(const psa_shape_t* s) {
  if (check_shape(s) != PSA_OK || s->dtype != PSA_DT_BF16) return 0;
  return bwd_layout(s).total;
}

psa_status_t psa_attention_bwd(const psa_shape_t* s, const void* q, const void* k, const void* v, const void* k_pyr,
                               const void* v_pyr, const uint8_t* mask, float sm_scale, const void* out,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv, void* ws,
                               size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  if (s->dtype != PSA_DT_BF16) return fail(PSA_ERR_UNSUPPORTED, "the backward pass takes bf16 tensors only");
  PSA_TRY(check_ptr(q, "q"));
  PSA_TRY(check_ptr(k, "k"));
  PSA_TRY(check_ptr(v, "v"));
  if (s->levels > 1) {
    PSA_TRY(check_ptr(k_pyr, "k_pyr"));
    PSA_TRY(check_ptr(v_pyr, "v_pyr"));
  }
  if (!mask) return fail(PSA_ERR_INVALID_ARG, "mask is NULL");
  PSA_TRY(check_ptr(out, "out"));
  PSA_TRY(check_ptr(lse, "lse"));
  PSA_TRY(check_ptr(dout, "dout"));
  PSA_TRY(check_ptr(dq, "dq"));
  PSA_TRY(check_ptr(dk, "dk"));
  PSA_TRY(check_ptr(dv, "dv"));
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return fail(PSA_ERR_INVALID_ARG, "sm_scale must be > 0");
  const BwdLayout L = bwd_layout(s);
  if (L.fwd.max_segs >= (1ll << 31) || L.fwd.max_tiles >= (1ll << 31) || L.max_entries >= (1ll << 31))
    return fail(PSA_ERR_UNSUPPORTED, "tile plan would exceed 2^31 entries");
  if (!ws || !aligned16(ws)) return fail(PSA_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
  if (ws_bytes < L.total) return fail(PSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const int64_t BHq = static_cast<int64_t>(s->B) * s->Hq, BHkv = static_cast<int64_t>(s->B) * s->Hkv;
  const char* kp = static_cast<const char*>(k_pyr);
  const char* vp = static_cast<const char*>(v_pyr);
  // tensor maps: for the dQ kernel Q and dO in 128-row boxes and the K / V
  // levels in the forward's segment boxes; for the dK / dV kernel Q and dO
  // in 64-row boxes and the K / V levels in 128-row boxes
  CUtensorMap mq[10], mkv[10];
  PSA_TRY(map3(&mq[0], q, BHq, s->N, s->d, 128));
  PSA_TRY(map3(&mq[1], dout, BHq, s->N, s->d, 128));
  PSA_TRY(map3(&mkv[0], q, BHq, s->N, s->d, 64));       // the dK / dV kernel streams 64-row query halves
  PSA_TRY(map3(&mkv[1], dout, BHq, s->N, s->d, 64));
  for (int l = 0; l < s->levels; ++l) {
    const void* kb = l == 0 ? k : static_cast<const void*>(kp + pyr_level_offset(s, l, 2));
    const void* vb = l == 0 ? v : static_cast<const void*>(vp + pyr_level_offset(s, l, 2));
    const int box = (s->block >> l) < 64 ? (s->block >> l) : 64;
    PSA_TRY(map3(&mq[2 + l], kb, BHkv, s->N >> l, s->d, box));
    PSA_TRY(map3(&mq[2 + s->levels + l], vb, BHkv, s->N >> l, s->d, box));
    PSA_TRY(map3(&mkv[2 + l], kb, BHkv, s->N >> l, s->d, 128));
    PSA_TRY(map3(&mkv[2 + s->levels + l], vb, BHkv, s->N >> l, s->d, 128));
  }
  const int nkb = static_cast<int>(ceil_div(s->N, s->block));
  // 1. the forward's tile plan (dQ walks it)
  psa::PlanArgs pa{};
  pa.B = s->B; pa.Hq = s->Hq; pa.N = s->N; pa.block = s->block; pa.nqb = nkb; pa.nkb = nkb;
  pa.levels = s->levels; pa.causal = s->causal != 0; pa.n_items = L.fwd.n_items; pa.mask = mask;
  pa.item_nseg = reinterpret_cast<int*>(w + L.fwd.nseg);
  pa.item_ntile = reinterpret_cast<int*>(w + L.fwd.ntile);
  pa.item_rows = reinterpret_cast<int*>(w + L.fwd.nrows);
  pa.item_seg_off = reinterpret_cast<int*>(w + L.fwd.seg_off);
  pa.item_tile_off = reinterpret_cast<int*>(w + L.fwd.tile_off);
  pa.tile_seg_off = reinterpret_cast<int*>(w + L.fwd.tile_seg_off);
  pa.segs = reinterpret_cast<int*>(w + L.fwd.segs);
  pa.queue = reinterpret_cast<int*>(w + L.fwd.queue);
  pa.hist = reinterpret_cast<int*>(w + L.fwd.hist);
  pa.n_hist = L.fwd.n_hist;
  pa.lpt_queue = 0;
  pa.stats = reinterpret_cast<long long*>(w + L.fwd.stats);
  PSA_CUDA(psa::launch_plan(pa, st), "plan launch");
  // 2. D = dO . O and lse in log2 units, padded
  float* lse2p = reinterpret_cast<float*>(w + L.lse2p);
  float* dpad = reinterpret_cast<float*>(w + L.dp);
  PSA_CUDA(psa::launch_bwd_prep(out, dout, lse, lse2p, dpad, BHq, s->N, s->d, L.fwd.n_qtiles, st), "prep launch");
  // 3. dQ
  psa::DqArgs qa{};
  qa.B = s->B; qa.Hq = s->Hq; qa.Hkv = s->Hkv; qa.N = s->N; qa.d = s->d; qa.block = s->block;
  qa.levels = s->levels; qa.causal = s->causal != 0; qa.n_items = L.fwd.n_items; qa.n_qtiles = L.fwd.n_qtiles;
  qa.scale_log2 = sm_scale * 1.4426950408889634f;
  qa.sm_scale = sm_scale;
  qa.item_tile_off = pa.item_tile_off;
  qa.item_rows = pa.item_rows;
  qa.tile_seg_off = pa.tile_seg_off;
  qa.segs = pa.segs;
  qa.queue = pa.queue;
  qa.lse2p = lse2p;
  qa.dp = dpad;
  qa.dq = dq;
  qa.status = reinterpret_cast<int*>(w + L.fwd.status);
  PSA_CUDA(psa::launch_dq(mq, qa, num_sms(), st), "dq launch");
  // 4. transposed plan, 5. dK^l / dV^l
  psa::TPlanArgs ta{};
  ta.B = s->B; ta.Hq = s->Hq; ta.Hkv = s->Hkv; ta.N = s->N; ta.block = s->block; ta.nqb = nkb; ta.nkb = nkb;
  ta.levels = s->levels; ta.causal = s->causal != 0; ta.n_qtiles = L.fwd.n_qtiles; ta.n_items = L.n_titems;
  for (int l = 0; l < 5; ++l) ta.level_base[l] = l <= s->levels ? L.level_base[l] : L.n_titems;
  for (int l = 0; l < 4; ++l) ta.level_tiles[l] = L.level_tiles[l];
  ta.mask = mask;
  ta.item_cnt = reinterpret_cast<int*>(w + L.tcnt);
  ta.item_off = reinterpret_cast<int*>(w + L.toff);
  ta.entry_qt = reinterpret_cast<int*>(w + L.eqt);
  ta.entry_mask = reinterpret_cast<unsigned*>(w + L.emask);
  PSA_CUDA(psa::launch_tplan(ta, st), "transposed plan launch");
  psa::DkvArgs ka{};
  ka.B = s->B; ka.Hq = s->Hq; ka.Hkv = s->Hkv; ka.N = s->N; ka.d = s->d; ka.block = s->block;
  ka.levels = s->levels; ka.causal = s->causal != 0; ka.n_qtiles = L.fwd.n_qtiles; ka.n_items = L.n_titems;
  for (int l = 0; l < 5; ++l) ka.level_base[l] = ta.level_base[l];
  for (int l = 0; l < 4; ++l) { ka.level_tiles[l] = L.level_tiles[l]; ka.level_off[l] = L.level_off[l]; }
  ka.scale_log2 = sm_scale * 1.4426950408889634f;
  ka.sm_scale = sm_scale;
  ka.item_off = ta.item_off;
  ka.entry_qt = ta.entry_qt;
  ka.entry_mask = ta.entry_mask;
  ka.lse2p = lse2p;
  ka.dp = dpad;
  ka.dkl = reinterpret_cast<float*>(w + L.dkl);
  ka.dvl = reinterpret_cast<float*>(w + L.dvl);
  ka.status = reinterpret_cast<int*>(w + L.fwd.status);
  PSA_CUDA(psa::launch_dkv(mkv, ka, num_sms(), st), "dkv launch");
  // 6. through the pooling of every level
  PSA_CUDA(psa::launch_pool_bwd(ka.dkl, L.level_off, dk, BHkv, s->N, s->d, s->levels, st), "pool backward (K)");
  PSA_CUDA(psa::launch_pool_bwd(ka.dvl, L.level_off, dv, BHkv, s->N, s->d, s->levels, st), "pool backward (V)");
  return PSA_OK;
}

psa_status_t psa_quantize_qk_fp8(const psa_shape_t* s, const void* q, const void* k, const void* k_pyr, uint8_t* q8,
                                 float* q_scale, uint8_t* k8, uint8_t* k8_pyr, float* k_scale, void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  if (s->dtype != PSA_DT_BF16) return fail(PSA_ERR_UNSUPPORTED, "the FP8 path takes bf16 tensors");
  PSA_TRY(check_ptr(q, "q"));
  PSA_TRY(check_ptr(k, "k"));
  PSA_TRY(check_ptr(q8, "q8"));
  PSA_TRY(check_ptr(q_scale, "q_scale"));
  PSA_TRY(check_ptr(k8, "k8"));
  PSA_TRY(check_ptr(k_scale, "k_scale"));
  if (s->levels > 1) {
    PSA_TRY(check_ptr(k_pyr, "k_pyr"));
    PSA_TRY(check_ptr(k8_pyr, "k8_pyr"));
  }
  size_t off[PSA_MAX_LEVELS] = {0, 0, 0, 0};
  for (int l = 1; l < s->levels; ++l) off[l] = pyr_level_offset(s, l, 1);
  const int64_t BHq = static_cast<int64_t>(s->B) * s->Hq, BHkv = static_cast<int64_t>(s->B) * s->Hkv;
  PSA_CUDA(psa::launch_quantize_qk_fp8(q, k, k_pyr, off, BHq, BHkv, s->N, s->d, s->levels, q8, q_scale, k8, k8_pyr,
                                       k_scale, static_cast<cudaStream_t>(stream)),
           "fp8 quantize launch");
  return PSA_OK;
}

size_t psa_attention_fp8_workspace_bytes(const psa_shape_t* s) {
  if (check_shape(s) != PSA_OK || s->dtype != PSA_DT_BF16 || s->d != 128) return 0;
  return fp8_layout(s).total;
}

psa_status_t psa_attention_fwd_fp8(const psa_shape_t* s, const void* q, const void* k, const void* v,
                                   const void* k_pyr, const void* v_pyr, const uint8_t* mask, float sm_scale,
                                   void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return attention_fp8(s, q, k, v, k_pyr, v_pyr, mask, sm_scale, out, lse, ws, ws_bytes, stream, false);
}

psa_status_t psa_attention_fwd_fp8_pv(const psa_shape_t* s, const void* q, const void* k, const void* v,
                                      const void* k_pyr, const void* v_pyr, const uint8_t* mask, float sm_scale,
                                      void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return attention_fp8(s, q, k, v, k_pyr, v_pyr, mask, sm_scale, out, lse, ws, ws_bytes, stream, true);
}

psa_status_t psa_attention_plan_stats(const psa_shape_t* s, const void* ws, int64_t* n_tiles, int64_t* n_rows,
                                      void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  if (!ws || !n_tiles || !n_rows) return fail(PSA_ERR_INVALID_ARG, "NULL argument");
  const AttnLayout L = attn_layout(s);
  long long st[2] = {0, 0};
  cudaStream_t str = static_cast<cudaStream_t>(stream);
  PSA_CUDA(cudaMemcpyAsync(st, static_cast<const char*>(ws) + L.stats, sizeof(st), cudaMemcpyDeviceToHost, str), "stats copy");
  PSA_CUDA(cudaStreamSynchronize(str), "stats sync");
  *n_tiles = st[0];
  *n_rows = st[1];
  return PSA_OK;
}

psa_status_t psa_get_device_status(void* ws, void* stream) {
  g_err[0] = 0;
  if (!ws) return fail(PSA_ERR_INVALID_ARG, "workspace is NULL");
  return read_status(ws, stream);
}

psa_status_t psa_debug_wait_control(void* ws, uint64_t limit_ns, int32_t trap, void* stream) {
  g_err[0] = 0;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 7u)) return fail(PSA_ERR_INVALID_ARG, "workspace is NULL or misaligned");
  struct {
    unsigned long long limit;
    int trap;
    int pad;
  } v = {limit_ns, trap ? 1 : 0, 0};
  static_assert(sizeof(v) == 16, "debug words");
  cudaStream_t str = static_cast<cudaStream_t>(stream);
  PSA_CUDA(cudaMemcpyAsync(static_cast<char*>(ws) + kWaitLimitOffset, &v, sizeof(v), cudaMemcpyHostToDevice, str),
           "debug word copy");
  PSA_CUDA(cudaStreamSynchronize(str), "debug word sync");
  return PSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ static workspace
// The workspace of psa_attention_fwd_static: one array per device, reserved
// when the library's device code is loaded.  Host code may not use the
// array's name as a pointer (it is a host-side shadow); the device address
// comes from cudaGetSymbolAddress, once per device, with that device current.
static __device__ __align__(256) unsigned char g_static_workspace[PSA_STATIC_WORKSPACE_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void* g_static_ptr[kMaxDevices] = {};

psa_status_t static_workspace(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(PSA_ERR_UNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress of the static workspace");
    // the header (status word, time-out record, wait limit) starts at zero;
    // afterwards only psa_get_static_device_status clears the status part
    e = cudaMemset(p, 0, 256);
    if (e != cudaSuccess) return cuda_fail(e, "static workspace header clear");
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return PSA_OK;
}
}  // namespace

extern "C" psa_status_t psa_get_static_device_status(void* stream) {
  g_err[0] = 0;
  void* ws = nullptr;
  PSA_TRY(static_workspace(&ws));
  return read_status(ws, stream);
}

extern "C" psa_status_t psa_attention_fwd_static(const psa_shape_t* s, const void* q, const void* k, const void* v,
                                                 const void* k_pyr, const void* v_pyr, const uint8_t* mask,
                                                 float sm_scale, void* out, float* lse, void* stream) {
  g_err[0] = 0;
  PSA_TRY(check_shape(s));
  const size_t need = attn_layout(s).total;
  if (need > PSA_STATIC_WORKSPACE_BYTES)
    return fail(PSA_ERR_WORKSPACE, "this shape needs a %zu-byte workspace; the static workspace holds %u bytes",
                need, PSA_STATIC_WORKSPACE_BYTES);
  // the remaining argument checks of psa_attention_fwd, so that nothing is
  // enqueued for a call that will be rejected
  PSA_TRY(check_ptr(q, "q"));
  PSA_TRY(check_ptr(k, "k"));
  PSA_TRY(check_ptr(v, "v"));
  PSA_TRY(check_ptr(out, "out"));
  if (s->levels > 1) {
    PSA_TRY(check_ptr(k_pyr, "k_pyr"));
    PSA_TRY(check_ptr(v_pyr, "v_pyr"));
  }
  if (!mask) return fail(PSA_ERR_INVALID_ARG, "mask is NULL");
  PSA_TRY(check_ptr(lse, "lse", false));
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return fail(PSA_ERR_INVALID_ARG, "sm_scale must be > 0");
  void* ws = nullptr;
  PSA_TRY(static_workspace(&ws));
  // the header was cleared once at set-up; a time-out stays recorded there
  // until psa_get_static_device_status reads it, and everything after the
  // header is rewritten by the plan of each call
  return psa_attention_fwd(s, q, k, v, k_pyr, v_pyr, mask, sm_scale, out, lse, ws, PSA_STATIC_WORKSPACE_BYTES,
                           stream);
}
