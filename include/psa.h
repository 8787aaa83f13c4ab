/*
 * psa.h -- C ABI of the Pyramid Sparse Attention (PSA) forward path on
 * NVIDIA B200 (sm_100a).
 *
 * The method (pages: "PSA: Pyramid Sparse Attention for Efficient Video
 * Understanding and Generation", summary article, section Method; the
 * "psa-pyramid-sparse-attention" skill page, sections Core Technique and
 * Implementation) has three steps, one entry point each:
 *
 *   psa_build_pyramid   KV pyramid: every KV block mean-pooled by 2, 4, 8
 *   psa_make_mask       per (query block, KV block) pair: a pyramid level
 *                       0..L-1 or SKIP, finer levels for more important pairs
 *   psa_attention_fwd   online-softmax attention of every query block over
 *                       its KV blocks, each read at its assigned level with a
 *                       +ln(2^l) logit bias
 *
 * and the gradients of the last step, psa_attention_bwd.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are contiguous row-major [B, H, N, d] in device memory, owned by
 *    the caller, base pointers 16-byte aligned.  Query head h reads KV head
 *    h / (Hq / Hkv).
 *  - The library never allocates device memory.  Scratch comes from the
 *    caller through a workspace pointer whose size the *_workspace_bytes
 *    query returns.  A workspace must be zero-filled once before its first
 *    use (it holds the device status word; see psa_get_device_status).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream.
 *  - Arguments are validated on the host before anything is launched; on a
 *    validation error nothing is written and the call returns
 *    PSA_ERR_INVALID_ARG, PSA_ERR_UNSUPPORTED or PSA_ERR_WORKSPACE.  A failed
 *    launch returns PSA_ERR_CUDA.  psa_last_error() then holds a message for
 *    the calling thread.
 *  - Supported set: dtype bf16 or fp32; d in {64, 128}; block in {64, 128};
 *    1 <= levels <= 4; block and N multiples of 2^(levels-1); Hq a multiple
 *    of Hkv; N >= 1; B*Hq*N*d < 2^31.  Anything else: PSA_ERR_UNSUPPORTED.
 *  - Device waits inside the kernels are bounded (about 2 s); a wait that
 *    runs out records PSA_ERR_TIMEOUT in the workspace status word and the
 *    kernel returns early instead of hanging.
 */
#ifndef PSA_H
#define PSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PSA_API __attribute__((visibility("default")))
#else
#define PSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PSA_OK = 0,
  PSA_ERR_INVALID_ARG = 1,   /* null pointer, size <= 0 (empty inputs included), bad enum, misaligned pointer */
  PSA_ERR_UNSUPPORTED = 2,   /* outside the supported set above */
  PSA_ERR_WORKSPACE = 3,     /* workspace null or smaller than the query says */
  PSA_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed */
  PSA_ERR_TIMEOUT = 5        /* a bounded device wait ran out (device status word) */
} psa_status_t;

typedef enum { PSA_DT_BF16 = 0, PSA_DT_FP32 = 1 } psa_dtype_t;

typedef enum {
  PSA_MASK_SAMPLE = 0,       /* generation task: sampled-query scoring */
  PSA_MASK_ANTIDIAG = 1,     /* understanding task: antidiagonal scoring */
  PSA_MASK_MEANKEY = 2       /* cheap scorer: block-mean queries against block-mean keys */
} psa_mask_mode_t;

typedef enum {
  PSA_POLICY_MASS = 0,       /* level = number of thresholds <= the exclusive prefix of the mass */
  PSA_POLICY_QUANTILE = 1    /* level = number of thresholds <= rank / visible blocks */
} psa_level_policy_t;

#define PSA_SKIP 0xFF
#define PSA_MAX_LEVELS 4
#define PSA_MAX_KV_BLOCKS 2048

/* Problem shape.  N is the unpadded token count; the last query/KV block may
 * be ragged.  causal != 0 hides keys after the query (a pooled token is
 * visible to query i iff the last token it averages is <= i). */
typedef struct {
  int32_t B, Hq, Hkv, N, d;
  int32_t block;             /* logical query and KV block size, tokens */
  int32_t levels;            /* L: pyramid levels 0..L-1 (pool 1, 2, 4, 8) */
  int32_t causal;
  int32_t dtype;             /* psa_dtype_t of q, k, v, pyramid and output */
} psa_shape_t;

/* Mask generator parameters (summary article, Method: sampling-based scores
 * for generation, antidiagonal scores plus an intra-block similarity check
 * for understanding; Results: threshold-based levels and a cosine condition
 * for pooling). */
typedef struct {
  int32_t mode;              /* psa_mask_mode_t */
  int32_t n_samples;         /* sampled queries per query block; must be 8 */
  int32_t stride;            /* antidiagonal stride S in {1, 2, 4, 8, 16}; block % S == 0 */
  float thresholds[8];       /* ascending cumulative-mass thresholds t_0..t_{L-1} */
  int32_t n_thresholds;      /* must equal shape.levels */
  float cos_min;             /* cosine gate; <= -2 disables it */
  int32_t n_dense_prefix;    /* tokens [0, n) are text: their blocks stay level 0 */
  float sm_scale;            /* softmax scale of the score; usually 1/sqrt(d) */
  int32_t policy;            /* psa_level_policy_t; 0 (the default when zeroed) = by mass */
} psa_mask_params_t;

/* ------------------------------------------------------------------------
 * Stage 1: KV pyramid (skill page, Core Technique / Implementation; summary
 * article, Method: repeated 1D mean pooling of every KV block).
 *
 * Level l (1 <= l < L) of K is [B, Hkv, N / 2^l, d]: token t is the mean of
 * input tokens t*2^l .. t*2^l + 2^l - 1, summed in fp32 and rounded once to
 * the shape's dtype (round to nearest even).  Levels 1..L-1 are stored back
 * to back in one buffer per tensor; psa_pyramid_level_offset gives where
 * level l starts (bytes, 16-byte aligned).  Level 0 is the input itself and
 * is not copied.
 *
 * blockcos (optional, may be NULL): fp32 [B, Hkv, nKB], nKB = ceil(N/block),
 * the mean pairwise cosine over i != j of the valid keys of each KV block
 * (a zero key counts as the zero vector; a one-key block gives 1).  It feeds
 * the cosine gate of psa_make_mask.
 * ------------------------------------------------------------------------ */
PSA_API size_t psa_pyramid_bytes(const psa_shape_t* shape);                   /* per tensor; 0 if L == 1 */
PSA_API size_t psa_pyramid_level_offset(const psa_shape_t* shape, int level); /* level in [1, L) */
PSA_API psa_status_t psa_build_pyramid(const psa_shape_t* shape, const void* k, const void* v,
                               void* k_pyr, void* v_pyr, float* blockcos, void* stream);

/* ------------------------------------------------------------------------
 * Stage 2: multi-level mask (summary article, Method and Results).
 *
 * Score, PSA_MASK_SAMPLE: query block I samples rows I*block + s*block/8,
 * s = 0..7 (rows >= N dropped); each sampled row takes a softmax of
 * sm_scale * q.k over all keys (keys <= the row when causal); the block
 * mass mass[I, J] is the mean over the samples of the probability falling
 * in KV block J.  Requires N % (block/8) == 0.
 * Score, PSA_MASK_ANTIDIAG: with stride S, A[a, c] = (sm_scale/S) *
 * sum_s q[a*S + S-1-s] . k[c*S + s]; softmax over key groups c (c <= a when
 * causal); mass[I, J] = mean over the query groups of I of the probability
 * in the key groups of J.  Requires N % S == 0.
 * Score, PSA_MASK_MEANKEY (skill page, Core Technique: a block scored by
 * the query against the mean of its keys): qbar_I and kbar_J are the means
 * of the valid tokens of query block I and key block J (fp64); mass[I, J] =
 * softmax over J of sm_scale * qbar_I . kbar_J (J <= I when causal).  It
 * reads Q and K once and needs no N alignment.
 * Levels, policy PSA_POLICY_MASS (summary article, Results: threshold-based
 * levels): per row (b, h, I) rank J by mass (descending, ties to lower J),
 * take the exclusive prefix C_J, level = #{t_l <= C_J}, SKIP when that count
 * reaches L.  Policy PSA_POLICY_QUANTILE (the rank-based alternative of the
 * same ablation): the block at rank r gets level #{t_l <= r / n_vis}, n_vis
 * = I + 1 when causal, else nKB; with L = 1 and t_0 = k / n_vis this keeps
 * the k heaviest blocks (a binary top-k mask).  Either policy with L = 1
 * gives a binary {0, SKIP} mask.  Then blocks holding a token <
 * n_dense_prefix (as query or key block) -> 0; if cos_min > -2 and level >=
 * 1 and blockcos[b, h_kv, J] < cos_min -> 0; if causal, J > I -> SKIP and
 * J == I -> 0.
 *
 * mask: uint8 [B, Hq, nQB, nKB] (PSA_SKIP = 0xFF).  mass_out (optional):
 * fp32 [B, Hq, nQB, nKB].  blockcos is required iff cos_min > -2.
 * nKB <= PSA_MAX_KV_BLOCKS.
 * ------------------------------------------------------------------------ */
PSA_API size_t psa_mask_workspace_bytes(const psa_shape_t* shape, const psa_mask_params_t* params);
PSA_API psa_status_t psa_make_mask(const psa_shape_t* shape, const psa_mask_params_t* params,
                           const void* q, const void* k, const float* blockcos,
                           uint8_t* mask, float* mass_out,
                           void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Stage 3: adaptive pyramid attention (summary article, Method: each KV
 * block fetched at its assigned level, a scale factor keeping the
 * probabilities consistent; news review, Methodology 4: plain scaled
 * dot-product attention over the selected pooled KV).
 *
 * For query token i in block I, over every KV block J with
 * l = mask[b, h, I, J] != SKIP and every pooled token p of J at level l:
 *   z_p = sm_scale * q_i . K^l[p] + l * ln 2,
 *   out_i = sum_p softmax(z)_p V^l[p],   lse_i = ln sum_p exp(z_p).
 * Under causal masking p is visible iff (p+1)*2^l - 1 <= i.  A row with no
 * visible key gets out = 0 and lse = -inf.  Rows >= N are not written.
 *
 * k_pyr/v_pyr: the buffers filled by psa_build_pyramid (NULL allowed iff
 * L == 1).  out: [B, Hq, N, d] in the shape's dtype.  lse (optional): fp32
 * [B, Hq, N], natural log.  For fp32 inputs the operands are rounded to
 * bf16 inside the workspace and the products are accumulated in fp32.
 * ------------------------------------------------------------------------ */
PSA_API size_t psa_attention_workspace_bytes(const psa_shape_t* shape);
PSA_API psa_status_t psa_attention_fwd(const psa_shape_t* shape, const void* q, const void* k, const void* v,
                               const void* k_pyr, const void* v_pyr, const uint8_t* mask,
                               float sm_scale, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * FP8 path of stage 3 (news review, Practical Implications, mentions mixed
 * FP16 / FP8 precision and nothing more; the scheme is this library's
 * reading).  The score product runs on e4m3 operands: each query row is
 * scaled by 448 / max|q_row| and every key of a KV head, at every pyramid
 * level, by 448 / max|K| over that head's level 0; scales and scaled
 * values are fp32, each rounded to the nearest e4m3 value (ties to even,
 * saturating at +-448).  The score of query i and pooled key p is then
 * sm_scale * q_scale[i] * k_scale[head] * (q8_i . k8_p) + l ln 2; V, the
 * probabilities (bf16) and the output (bf16) are as in psa_attention_fwd.
 * bf16 tensors with d = 128 only (else PSA_ERR_UNSUPPORTED).  The
 * rounding of Q and K costs accuracy: on the presets' inputs the output
 * moves by up to about 0.1 (mean about 0.01) from the bf16 path's.
 *
 * psa_quantize_qk_fp8: q -> q8 codes [B, Hq, N, d] (one byte each) and
 * q_scale fp32 [B, Hq, N]; k (level 0) and the levels of k_pyr -> k8
 * [B, Hkv, N, d] and k8_pyr (levels 1..L-1 back to back, one byte per
 * element, level l at the element offset psa_pyramid_level_offset gives
 * divided by 2), and k_scale fp32 [B, Hkv].  psa_attention_fwd_fp8 does
 * the same into its workspace (psa_attention_fp8_workspace_bytes), then
 * the attention.
 * ------------------------------------------------------------------------ */
PSA_API psa_status_t psa_quantize_qk_fp8(const psa_shape_t* shape, const void* q, const void* k, const void* k_pyr,
                                         uint8_t* q8, float* q_scale, uint8_t* k8, uint8_t* k8_pyr,
                                         float* k_scale, void* stream);
PSA_API size_t psa_attention_fp8_workspace_bytes(const psa_shape_t* shape);
PSA_API psa_status_t psa_attention_fwd_fp8(const psa_shape_t* shape, const void* q, const void* k, const void* v,
                                           const void* k_pyr, const void* v_pyr, const uint8_t* mask,
                                           float sm_scale, void* out, float* lse,
                                           void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * psa_attention_fwd_fp8_pv: the FP8 path with the probabilities and values
 * in e4m3 as well (the same pages; this library's reading), so both
 * products of the attention run on 8-bit operands.  Q and K as in
 * psa_attention_fwd_fp8.  Every value of a KV head, at every pyramid
 * level, is scaled by 448 / max|V| over that head's level 0 and rounded
 * like the keys.  The probabilities of a query row are P_p = 2^(a_p - r)
 * with a_p the logit in log2 units and r a whole number at or above the
 * largest a_p seen so far (moved only when the maximum grows by more than
 * 5), computed in fp32 and rounded to e4m3; because e4m3 is a floating
 * format the rounded values do not depend on r while they stay in its
 * normal range.  The output is v_scale[head] * sum_p e4m3(P_p) v8_p /
 * sum_p P_p (the normaliser sums the unrounded fp32 probabilities); lse as
 * in psa_attention_fwd.  Arguments, workspace (the same size as
 * psa_attention_fwd_fp8's), layouts and errors as psa_attention_fwd_fp8;
 * the values are coded into the workspace like the keys.
 * ------------------------------------------------------------------------ */
PSA_API psa_status_t psa_attention_fwd_fp8_pv(const psa_shape_t* shape, const void* q, const void* k, const void* v,
                                              const void* k_pyr, const void* v_pyr, const uint8_t* mask,
                                              float sm_scale, void* out, float* lse,
                                              void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Backward pass of stage 3 (the pages give none; news review, Methodology
 * 4, says the model trains end to end through the pooled attention, and the
 * summary article, Results, pairs PSA with distillation).  The derivative
 * of psa_attention_fwd's definition with the mask held fixed: with
 * P = exp(z - lse) over the row's key set, dP = dO . V^l[p], D = dO . O and
 * dZ = P (dP - D),
 *   dq_i = sm_scale sum_p dZ_ip K^l[p],
 *   dK^l[p] = sm_scale sum_i dZ_ip q_i,   dV^l[p] = sum_i P_ip dO_i,
 * and through the pooling (level l token t is the mean of input tokens
 * t 2^l .. t 2^l + 2^l - 1):  dk[t] = sum_l dK^l[t >> l] / 2^l, same for v.
 *
 * Inputs: the forward's q, k, v, pyramid buffers, mask and sm_scale, its
 * output `out` and its lse (both required), and dout = dL/dout; all
 * [B, H, N, d] bf16 except lse (fp32 [B, Hq, N]).  Outputs dq [B, Hq, N, d],
 * dk and dv [B, Hkv, N, d], bf16, fully overwritten (rows with no visible
 * key get dq = 0; KV tokens no query uses get 0).  Products are bf16 with
 * fp32 accumulation; P and dZ are rounded to bf16 before their products,
 * dK^l and dV^l are summed in fp32 before the pooling backward.  bf16
 * tensors only (fp32 shapes: PSA_ERR_UNSUPPORTED).  The workspace (size
 * from psa_attention_bwd_workspace_bytes) holds the forward's tile plan,
 * the transposed plan of the dK / dV kernel and the fp32 level gradients;
 * like every workspace it is zero-filled once before first use and carries
 * the status word read by psa_get_device_status.
 * ------------------------------------------------------------------------ */
PSA_API size_t psa_attention_bwd_workspace_bytes(const psa_shape_t* shape);
PSA_API psa_status_t psa_attention_bwd(const psa_shape_t* shape, const void* q, const void* k, const void* v,
                                       const void* k_pyr, const void* v_pyr, const uint8_t* mask,
                                       float sm_scale, const void* out, const float* lse, const void* dout,
                                       void* dq, void* dk, void* dv,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* psa_attention_fwd without a workspace argument, for callers that cannot
 * allocate device memory themselves: for example a plugin inside a host
 * framework that owns every device allocation, or a latency-critical loop
 * where cudaMalloc's implicit device synchronisation is not acceptable.  The
 * pages have no counterpart; this is an interface convenience only.
 *
 * The workspace is a file-scope device array of PSA_STATIC_WORKSPACE_BYTES
 * (32 MiB) inside libpsa.so; every GPU that loads the library holds it until
 * the process exits.  Shapes whose psa_attention_workspace_bytes exceeds it
 * are rejected with PSA_ERR_WORKSPACE before anything is launched (it covers,
 * for example, the Qwen2.5-VL- and Wan2.1-1.3B-shaped problems, not the
 * Wan2.1-14B-shaped one).  The first call on each device (of this function or
 * of psa_get_static_device_status) looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and zero-fills its
 * 256-byte header with a synchronous cudaMemset, so make that first call
 * before any stream capture.  No device memory is allocated or freed.  All
 * calls share the one array and it keeps the last call's contents; calls
 * that overlap on the GPU (other streams, other threads) race on the array.
 * A bounded-wait time-out in the kernel is recorded in the array's status
 * word and stays there, across later calls, until
 * psa_get_static_device_status reads and clears it. */
#define PSA_STATIC_WORKSPACE_BYTES (32u << 20)
PSA_API psa_status_t psa_attention_fwd_static(const psa_shape_t* shape, const void* q, const void* k,
                                              const void* v, const void* k_pyr, const void* v_pyr,
                                              const uint8_t* mask, float sm_scale, void* out, float* lse,
                                              void* stream);

/* psa_get_device_status for the static workspace of
 * psa_attention_fwd_static on the current device: reads (synchronising on
 * `stream`) and clears its status word and time-out record. */
PSA_API psa_status_t psa_get_static_device_status(void* stream);

/* Executed work of the last plan built in `workspace` by psa_attention_fwd:
 * fills (synchronising on `stream`) the number of 128-row KV tiles and the
 * number of KV rows that hold real (non-padding) pooled tokens. */
PSA_API psa_status_t psa_attention_plan_stats(const psa_shape_t* shape, const void* workspace,
                                      int64_t* n_tiles, int64_t* n_rows, void* stream);

/* Reads the device status word of a workspace (synchronising on `stream`)
 * and clears it: PSA_OK, or PSA_ERR_TIMEOUT if a bounded wait ran out in a
 * kernel that used this workspace since the last read.  On a time-out,
 * psa_last_error() names the wait that gave up first (its site number, CTA,
 * thread and progress counters).  The status word and that record occupy
 * the first 36 bytes of every workspace. */
PSA_API psa_status_t psa_get_device_status(void* workspace, void* stream);

/* Debug and test aid for the time-out path of the attention kernel when it
 * runs on `workspace` (the pages have no counterpart).  With trap != 0,
 * every CTA waits once, right after its first K load, on a barrier that no
 * thread arrives at; that wait gives up after limit_ns nanoseconds (0: the
 * built-in 2 s), long before any other wait of the kernel could, so the
 * CTA raises its abort flag, every role unwinds, the copies and MMAs in
 * flight are drained, TMEM is freed, and psa_get_device_status returns
 * PSA_ERR_TIMEOUT naming wait site 10.  The call's outputs are then
 * incomplete.  The two values sit at bytes 40..51 of the workspace header
 * and outlive psa_get_device_status, which clears only the first 36 bytes;
 * call again with trap = 0 to restore normal operation.  Synchronises on
 * `stream`.  `workspace` must be 8-byte aligned. */
PSA_API psa_status_t psa_debug_wait_control(void* workspace, uint64_t limit_ns, int32_t trap, void* stream);

/* Message of the last failed call on this thread ("" if none). */
PSA_API const char* psa_last_error(void);

/* ABI version: 100 * major + minor. */
PSA_API int32_t psa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PSA_H */
