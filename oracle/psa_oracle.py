"""CPU oracle for the Pyramid Sparse Attention (PSA) forward path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  The product path (``video_transformers_b200``) never calls it,
and this module imports nothing from the product path: the two share no
kernels, headers, helpers, tables or constants.

Everything here is plain numpy in float64.  Inputs arrive as whatever the
CUDA path was given (fp32 or bf16 tensors), converted exactly to float64.
The code follows the definitions as written, with no blocking, fusion or
reordering beyond what the definition states, so it can be read against the
pages line by line.

Pages cited (title, then section):
  [skill]    "psa-pyramid-sparse-attention" skill page: "Core Technique",
             "Implementation" (pooled KV cache creation).
  [article]  "PSA: Pyramid Sparse Attention for Efficient Video Understanding
             and Generation", summary article: "Problem", "Method", "Results".
  [news]     "[Paper] PSA: Pyramid Sparse Attention ..." news review:
             "Methodology" items 2 and 4.
  [abstract] the arXiv abstract of the same paper.

Readings taken where the pages are silent (each is also listed with its
reason in the design notes):
  R1  consistency scale = +ln(2^l) logit bias for a level-l pooled token
      (equivalent to repeating the pooled token 2^l times, which is how
      [news] Methodology 4 describes pooled KV being brought back to size).
  R2  sm_scale defaults to 1/sqrt(d) ([news] Methodology 4 combines the
      query with the selected KV by ordinary scaled dot-product attention).
  R3  causal visibility of a pooled token: visible to query i iff the last
      token it averages is <= i.
  R4  a query row with no visible key gets o = 0, lse = -inf.
  R5  sampling score: 8 evenly strided rows per query block
      (row = I*block + s*block/8), softmax over all valid keys at full
      resolution (keys <= i when causal), block-summed, averaged over the
      valid samples.
  R6  antidiagonal score with stride S: per S-group, the mean logit along
      the antidiagonal of the S x S sub-tile; softmax over key groups
      (c <= a when causal); block-summed; averaged over the query groups of
      the block.
  R7  level assignment: rank blocks by mass (descending, ties to the lower
      index), exclusive prefix C_J, level = #{t_l <= C_J}, SKIP when that
      count reaches L.
  R8  forced rules, applied in this order after R7: blocks holding any token
      below n_dense_prefix (as query or key block) -> level 0; cosine gate
      (level >= 1 and blockcos < cos_min -> level 0); causal: J > I -> SKIP,
      J == I -> level 0.
  R9  block cosine = mean pairwise cosine over i != j of the block's valid
      keys; a zero key has unit vector 0; a one-key block scores 1.
  R10 quantile (rank) level assignment, the alternative to R7 that the
      [article] Results ablation compares with: rank as in R7; the block at
      rank r gets level #{t_l <= r / n_vis}, SKIP when that count reaches L,
      where n_vis is the number of key blocks the row can see (J <= I when
      causal, else all).  With L = 1 and t_0 = k / n_vis this keeps exactly
      the k heaviest blocks (a top-k binary mask).
  R11 mean-key score ([skill] Core Technique, block importance as the
      query against the mean of the block's keys): the query side is the
      mean of the query block's valid queries as well; mass[I, J] =
      softmax over visible J of sm_scale * mean_q(I) . mean_k(J).
  R12 backward pass: the mask (the levels) is a fixed selection and is not
      differentiated; gradients flow through the pooling of each level as a
      mean (1/2^l to each averaged token).
  R13 FP8 path ([news] Practical Implications mentions mixed FP16/FP8
      precision and nothing more): the query and key operands of the score
      product are rounded to e4m3 (3 mantissa bits, largest value 448,
      nearest value with ties to even, saturating).  Each query row is
      scaled by 448 / max|q_row|; every key of a KV head, at every pyramid
      level, by 448 / max|K| over that head's level 0 (a mean is no larger
      than the largest of its terms, so no level saturates).  Scales and
      the scaled values are computed in fp32; the score is the product of
      the e4m3 values times both scales.  Values and probabilities stay as
      in R1-R4.
  R14 FP8 probabilities and values (the rest of the FP8 path; the pages say
      no more than R13 does): the values of every level are rounded to e4m3
      with one scale per KV head from level 0, as the keys in R13.  The
      probabilities of a query row are P_p = 2^(a_p - M) with a_p = z_p /
      ln 2 the logit in log2 units and M = ceil(max_p a_p), computed in fp32
      and rounded to e4m3; the output is sum_p e4m3(P_p) V_p / sum_p P_p
      (the normaliser sums the unrounded P), and lse is as in R1-R4.  e4m3
      is a floating format, so moving M by a whole number of binades moves
      every rounded P by the same power of two while the values stay in
      its normal range (>= 2^-6): an online implementation whose running
      reference is a whole number of binades at or below M rounds the same
      values.  It differs only for probabilities that are below 2^-6 at
      one reference and not at the other.

Pins: every function here is checked by ``tests/test_oracle_pins.py``
against closed forms, invariants, brute force or an independent library
routine; see that file's header for which pin covers which function.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

SKIP = 0xFF
LN2 = math.log(2.0)


def _f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor (fp32/bf16) or array to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ======================================================================================
# Stage 1: KV pyramid
# ======================================================================================

def pool_level(x, level: int) -> np.ndarray:
    """Level ``level`` of the KV pyramid: every run of g = 2^level consecutive
    tokens replaced by its mean ([skill] Core Technique, level l holds the
    KV pooled by 2^l; [skill] Implementation, average pooling over tokens by
    a factor 2**level taken from the full-resolution cache; [article] Method,
    the pyramid comes from repeated one-dimensional mean pooling).

    x: [B, H, N, d] -> [B, H, N / g, d].  The direct mean equals the
    progressive (pairwise) pooling in exact arithmetic.  N must be a
    multiple of g, so groups never straddle the end of the sequence."""
    x = _f64(x)
    B, H, N, d = x.shape
    g = 1 << level
    if N % g:
        raise ValueError("sequence length must be a multiple of the pooling factor")
    return x.reshape(B, H, N // g, g, d).mean(axis=3)


def build_pyramid(k, v, levels: int) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Levels 0..L-1 of K and V; level 0 is the input itself ([skill]
    Core Technique, level 0 is the unpooled KV)."""
    kp = [_f64(k)] + [pool_level(k, l) for l in range(1, levels)]
    vp = [_f64(v)] + [pool_level(v, l) for l in range(1, levels)]
    return kp, vp


def block_cosine(k, block: int) -> np.ndarray:
    """Intra-block similarity statistic used by the pooling constraint
    ([article] Method, the understanding-task scorer checks similarity inside
    each block; [article] Results, a cosine-similarity condition decides
    whether a block may be pooled).  Reading R9: the
    mean over ordered pairs i != j of cos(k_i, k_j) over the valid keys of
    block J, brute force over all pairs.

    k: [B, H, N, d] -> [B, H, nKB]."""
    k = _f64(k)
    B, H, N, d = k.shape
    nkb = -(-N // block)
    out = np.empty((B, H, nkb))
    for b in range(B):
        for h in range(H):
            for J in range(nkb):
                keys = k[b, h, J * block:min((J + 1) * block, N)]
                n = keys.shape[0]
                if n == 1:
                    out[b, h, J] = 1.0
                    continue
                norms = np.sqrt((keys * keys).sum(axis=1))
                unit = np.where(norms[:, None] > 0, keys / np.where(norms > 0, norms, 1.0)[:, None], 0.0)
                total = 0.0
                for i in range(n):
                    cos_i = unit @ unit[i]
                    total += cos_i.sum() - cos_i[i]
                out[b, h, J] = total / (n * (n - 1))
    return out


# ======================================================================================
# Stage 2: multi-level mask
# ======================================================================================

def _softmax_rows(z: np.ndarray) -> np.ndarray:
    """Row softmax with the max subtracted; rows that are all -inf give 0."""
    m = z.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(z - m)
    s = e.sum(axis=1, keepdims=True)
    return np.where(s > 0, e / np.where(s > 0, s, 1.0), 0.0)


def _block_sum(p: np.ndarray, width: int, nblocks: int) -> np.ndarray:
    """Sum the columns of p in consecutive runs of ``width`` (last run ragged)."""
    rows, cols = p.shape
    pad = nblocks * width - cols
    if pad:
        p = np.concatenate([p, np.zeros((rows, pad))], axis=1)
    return p.reshape(rows, nblocks, width).sum(axis=2)


def sampling_rows(I: int, block: int, N: int, n_samples: int = 8) -> List[int]:
    """Reading R5: the sampled query rows of block I."""
    step = block // n_samples
    return [I * block + s * step for s in range(n_samples) if I * block + s * step < N]


def sampling_mass(q, k, block: int, sm_scale: float, causal: bool = False, n_samples: int = 8,
                  rows: Optional[Iterable[Tuple[int, int, int]]] = None) -> np.ndarray:
    """Block importance by sampling ([article] Method, the generation-task
    scorer samples queries).  Reading R5.

    q: [B, Hq, N, d], k: [B, Hkv, N, d].  Returns mass [B, Hq, nQB, nKB];
    when ``rows`` lists (b, h, I) triples only those rows are filled (the
    rest stay NaN)."""
    q = _f64(q)
    k = _f64(k)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    nb = -(-N // block)
    mass = np.full((B, Hq, nb, nb), np.nan)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nb)]
    for b, h, I in rows:
        keys = k[b, h // grp]
        r = sampling_rows(I, block, N, n_samples)
        z = sm_scale * (q[b, h, r] @ keys.T)                       # [ns, N]
        if causal:
            j = np.arange(N)
            z = np.where(j[None, :] <= np.asarray(r)[:, None], z, -np.inf)
        p = _softmax_rows(z)
        mass[b, h, I] = _block_sum(p, block, nb).mean(axis=0)
    return mass


def antidiag_logits(qh: np.ndarray, kh: np.ndarray, stride: int, sm_scale: float) -> np.ndarray:
    """Reading R6 of the understanding-task score ([article] Method, scores
    come from antidiagonals): for query group a and key group c,
    A[a, c] = (sm_scale / S) * sum_{s<S} q[a*S + S-1-s] . k[c*S + s].

    qh, kh: [N, d] (one head); returns [N/S, N/S]."""
    N, d = qh.shape
    S = stride
    G = N // S
    A = np.zeros((G, G))
    for s in range(S):
        A += qh[np.arange(G) * S + (S - 1 - s)] @ kh[np.arange(G) * S + s].T
    return (sm_scale / S) * A


def antidiag_mass(q, k, block: int, stride: int, sm_scale: float, causal: bool,
                  rows: Optional[Iterable[Tuple[int, int, int]]] = None) -> np.ndarray:
    """Block importance from antidiagonal scores (reading R6): group
    probabilities P[a, :] = softmax_c A[a, c] (c <= a when causal), then
    mass[I, J] = mean over the query groups a of block I of sum over the key
    groups c of block J of P[a, c]."""
    q = _f64(q)
    k = _f64(k)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    S = stride
    if N % S:
        raise ValueError("sequence length must be a multiple of the stride")
    G = N // S
    gpb = block // S
    nb = -(-N // block)
    mass = np.full((B, Hq, nb, nb), np.nan)
    want = None if rows is None else {}
    if rows is not None:
        for b, h, I in rows:
            want.setdefault((b, h), []).append(I)
    for b in range(B):
        for h in range(Hq):
            if want is not None and (b, h) not in want:
                continue
            A = antidiag_logits(q[b, h], k[b, h // grp], S, sm_scale)
            if causal:
                a = np.arange(G)
                A = np.where(a[None, :] <= a[:, None], A, -np.inf)
            P = _softmax_rows(A)
            per_group = _block_sum(P, gpb, nb)                       # [G, nb]
            Is = range(nb) if want is None else want[(b, h)]
            for I in Is:
                mass[b, h, I] = per_group[I * gpb:min((I + 1) * gpb, G)].mean(axis=0)
    return mass


def assign_levels_row(mass_row: Sequence[float], thresholds: Sequence[float], levels: int) -> np.ndarray:
    """Threshold-based multi-level assignment for one query block ([article]
    Method, finer levels for critical blocks, coarser for less important
    ones, the least important skipped entirely; [article] Results, the
    ablation favours thresholds for building the mask).  Reading R7."""
    mass_row = np.asarray(mass_row, dtype=np.float64)
    n = mass_row.shape[0]
    order = sorted(range(n), key=lambda J: (-mass_row[J], J))
    out = np.empty(n, dtype=np.int64)
    C = 0.0
    for J in order:
        lev = sum(1 for t in thresholds if t <= C)
        out[J] = SKIP if lev >= levels else lev
        C += mass_row[J]
    return out


def exclusive_prefix(mass_row: Sequence[float]) -> np.ndarray:
    """C_J of reading R7 for every J (used by the ambiguity band)."""
    mass_row = np.asarray(mass_row, dtype=np.float64)
    order = sorted(range(mass_row.shape[0]), key=lambda J: (-mass_row[J], J))
    C = np.empty_like(mass_row)
    acc = 0.0
    for J in order:
        C[J] = acc
        acc += mass_row[J]
    return C


def assign_levels_quantile_row(mass_row: Sequence[float], thresholds: Sequence[float], levels: int,
                               n_visible: Optional[int] = None) -> np.ndarray:
    """Rank-based (quantile / top-k) level assignment for one query block,
    the alternative the [article] Results ablation weighs against threshold
    levels.  Reading R10: the block at rank r (mass descending, ties to the
    lower index) gets level #{t_l <= r / n_visible}."""
    mass_row = np.asarray(mass_row, dtype=np.float64)
    n = mass_row.shape[0]
    nv = n if n_visible is None else n_visible
    order = sorted(range(n), key=lambda J: (-mass_row[J], J))
    out = np.empty(n, dtype=np.int64)
    for r, J in enumerate(order):
        frac = r / nv
        lev = sum(1 for t in thresholds if t <= frac)
        out[J] = SKIP if lev >= levels else lev
    return out


def block_means(x, block: int) -> np.ndarray:
    """[B, H, N, d] -> [B, H, nB, d]: the mean of each block's valid tokens
    (the last block may be ragged)."""
    x = _f64(x)
    B, H, N, d = x.shape
    nb = -(-N // block)
    out = np.empty((B, H, nb, d))
    for J in range(nb):
        out[:, :, J] = x[:, :, J * block:min((J + 1) * block, N)].mean(axis=2)
    return out


def meankey_mass(q, k, block: int, sm_scale: float, causal: bool = False,
                 rows: Optional[Iterable[Tuple[int, int, int]]] = None) -> np.ndarray:
    """Block importance from block means ([skill] Core Technique, a block is
    scored by the query against the mean of its keys).  Reading R11.
    Returns mass [B, Hq, nQB, nKB]; rows not listed in ``rows`` stay NaN."""
    qm = block_means(q, block)
    km = block_means(k, block)
    B, Hq, nb, d = qm.shape
    grp = Hq // km.shape[1]
    mass = np.full((B, Hq, nb, nb), np.nan)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nb)]
    for b, h, I in rows:
        z = sm_scale * (km[b, h // grp] @ qm[b, h, I])             # [nKB]
        if causal:
            z = np.where(np.arange(nb) <= I, z, -np.inf)
        mass[b, h, I] = _softmax_rows(z[None, :])[0]
    return mass


def apply_forced_rules(levels_row: np.ndarray, I: int, block: int, levels: int, causal: bool,
                       n_dense_prefix: int = 0, cos_row: Optional[np.ndarray] = None,
                       cos_min: float = -3.0) -> np.ndarray:
    """Reading R8."""
    out = levels_row.copy()
    n = out.shape[0]
    for J in range(n):
        if n_dense_prefix > 0 and (I * block < n_dense_prefix or J * block < n_dense_prefix):
            out[J] = 0
        if cos_row is not None and cos_min > -2.0 and out[J] != SKIP and out[J] >= 1 \
                and cos_row[J] < cos_min:
            out[J] = 0
        if causal:
            if J > I:
                out[J] = SKIP
            elif J == I:
                out[J] = 0
    return out


def make_mask(mass: np.ndarray, thresholds, levels: int, block: int, causal: bool,
              n_dense_prefix: int = 0, blockcos: Optional[np.ndarray] = None, cos_min: float = -3.0,
              hq_per_kv: int = 1, rows=None, policy: str = "mass") -> np.ndarray:
    """mass [B,Hq,nQB,nKB] -> mask uint8 of the same shape (SKIP = 0xFF).
    policy "mass": levels by reading R7; "quantile": by reading R10."""
    B, Hq, nqb, nkb = mass.shape
    out = np.full((B, Hq, nqb, nkb), SKIP, dtype=np.int64)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nqb)]
    for b, h, I in rows:
        if policy == "quantile":
            lev = assign_levels_quantile_row(mass[b, h, I], thresholds, levels,
                                             min(I + 1, nkb) if causal else nkb)
        else:
            lev = assign_levels_row(mass[b, h, I], thresholds, levels)
        cos_row = None if blockcos is None else blockcos[b, h // hq_per_kv]
        out[b, h, I] = apply_forced_rules(lev, I, block, levels, causal, n_dense_prefix, cos_row, cos_min)
    return out.astype(np.uint8)


def ambiguous_pairs(mass: np.ndarray, thresholds, eps: float = 1e-6, rows=None,
                    blockcos: Optional[np.ndarray] = None, cos_min: float = -3.0,
                    hq_per_kv: int = 1) -> np.ndarray:
    """Pairs whose level may legitimately differ between an fp32 and an fp64
    evaluation: some threshold t lies within eps of the range of C_J that
    near-equal masses (relative eps) allow, or the block cosine lies within
    eps of cos_min.  Computed from the oracle's masses."""
    B, Hq, nqb, nkb = mass.shape
    amb = np.zeros(mass.shape, dtype=bool)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nqb)]
    for b, h, I in rows:
        m = mass[b, h, I]
        for J in range(nkb):
            lo = m[m > m[J] * (1 + eps)].sum()
            hi = m[m >= m[J] * (1 - eps)].sum() - m[J]
            for t in thresholds:
                if lo - eps <= t <= hi + eps:
                    amb[b, h, I, J] = True
            if blockcos is not None and cos_min > -2.0 and abs(blockcos[b, h // hq_per_kv, J] - cos_min) <= eps:
                amb[b, h, I, J] = True
    return amb


def ambiguous_pairs_quantile(mass: np.ndarray, thresholds, levels: int, causal: bool, eps: float = 1e-6,
                             rows=None) -> np.ndarray:
    """Pairs whose rank-based level (reading R10) may legitimately differ
    between an fp32 and an fp64 evaluation: the ranks that near-equal masses
    (relative eps) allow for block J span a level boundary."""
    B, Hq, nqb, nkb = mass.shape
    amb = np.zeros(mass.shape, dtype=bool)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nqb)]
    for b, h, I in rows:
        m = mass[b, h, I]
        nv = min(I + 1, nkb) if causal else nkb
        for J in range(nkb):
            r_lo = int((m > m[J] * (1 + eps)).sum())
            r_hi = int((m >= m[J] * (1 - eps)).sum()) - 1
            lev = {sum(1 for t in thresholds if t <= r / nv) for r in (r_lo, r_hi)}
            if len(lev) > 1:
                amb[b, h, I, J] = True
    return amb


# ======================================================================================
# FP8 (e4m3) query / key operands, reading R13
# ======================================================================================

E4M3_MAX = 448.0


def e4m3_codes(x32) -> np.ndarray:
    """The e4m3 byte of each fp32 value: nearest e4m3 value, ties to even,
    saturating at +-448 (the clip; the cast of an in-range value is the
    library's round-to-nearest-even conversion)."""
    import torch
    t = torch.as_tensor(np.clip(np.asarray(x32, dtype=np.float32), -E4M3_MAX, E4M3_MAX))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_values(codes) -> np.ndarray:
    """float64 value of each e4m3 byte."""
    import torch
    return torch.as_tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _fp32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float32)


def _scale_and_inverse(am: np.ndarray):
    """fp32 dequantization scale max/448 and quantization multiplier 448/max
    (0 and 0 for an all-zero row or head)."""
    am = am.astype(np.float32)
    nz = am > 0
    inv = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, am, np.float32(1)), np.float32(0)).astype(np.float32)
    scale = (am / np.float32(E4M3_MAX)).astype(np.float32)
    return scale, inv


def quantize_rows_e4m3(x):
    """Reading R13 for the query side: x [B, H, N, d] -> (codes uint8
    [B, H, N, d], scale fp32 [B, H, N]); row value = e4m3 value * scale."""
    xf = _fp32(x)
    am = np.abs(xf).max(axis=-1)
    scale, inv = _scale_and_inverse(am)
    codes = e4m3_codes((xf * inv[..., None]).astype(np.float32))
    return codes, scale


def quantize_heads_e4m3(levels):
    """Reading R13 for the key side: levels = [K (level 0), K^1, ...], each
    [B, H, n_l, d] -> (codes per level, scale fp32 [B, H]) with one scale
    per head from level 0's largest magnitude."""
    l0 = _fp32(levels[0])
    am = np.abs(l0).reshape(l0.shape[0], l0.shape[1], -1).max(axis=-1)
    scale, inv = _scale_and_inverse(am)
    codes = [e4m3_codes((_fp32(x) * inv[:, :, None, None]).astype(np.float32)) for x in levels]
    return codes, scale


def attention_fp8(q, kp, vp, mask, block: int, sm_scale: float, causal: bool, rows=None, pv: bool = False):
    """Adaptive pyramid attention (as :func:`attention`) with the query rows
    and the key levels replaced by their e4m3 values times their scales
    (reading R13); values, bias and softmax unchanged.  With ``pv`` the
    value levels are rounded to e4m3 as the keys and the probabilities as
    in reading R14.  kp / vp: the levels as the attention receives them
    (level 0 first)."""
    qc, qs = quantize_rows_e4m3(q)
    kc, ks = quantize_heads_e4m3(kp)
    qd = e4m3_values(qc) * qs.astype(np.float64)[..., None]
    kd = [e4m3_values(c) * ks.astype(np.float64)[:, :, None, None] for c in kc]
    if pv:
        vc, vs = quantize_heads_e4m3(vp)
        vd = [e4m3_values(c) * vs.astype(np.float64)[:, :, None, None] for c in vc]
        return attention(qd, kd, vd, mask, block, sm_scale, causal, rows=rows, p_e4m3=True)
    return attention(qd, kd, [_f64(x) for x in vp], mask, block, sm_scale, causal, rows=rows)


def softmax_pv_e4m3(z, vals) -> np.ndarray:
    """Reading R14 for a set of query rows: z [r, n] natural-log logits
    (-inf where masked), vals [n, d].  a = z / ln 2, M = ceil(max a) per
    row, P = 2^(a - M) in fp32, rounded to e4m3; returns
    sum e4m3(P) vals / sum P per row (rows with no visible key: 0)."""
    z = np.asarray(z, dtype=np.float64)
    a = z / LN2
    amax = a.max(axis=1, keepdims=True) if a.shape[1] else np.full((a.shape[0], 1), -np.inf)
    empty = ~np.isfinite(amax)
    M = np.where(empty, 0.0, np.ceil(np.where(empty, 0.0, amax)))
    p = np.exp2(a - M).astype(np.float32)
    pq = e4m3_values(e4m3_codes(p))
    den = p.astype(np.float64).sum(axis=1, keepdims=True)
    out = (pq @ np.asarray(vals, dtype=np.float64)) / np.where(den > 0, den, 1.0)
    return np.where(empty, 0.0, out)


# ======================================================================================
# Stage 3: adaptive pyramid attention
# ======================================================================================

def level_bias(level: int) -> float:
    """Reading R1 of the consistency scale ([article] Method, a scale factor
    keeps the attention probabilities consistent across levels):
    a level-l pooled token stands for 2^l tokens, so its logit gets +ln(2^l)."""
    return level * LN2


def gather_keys(kp, vp, mask_row: Sequence[int], block: int, N: int, b: int, hk: int):
    """The key set of one query block ([article] Method, each KV block is
    read at the pyramid level the mask assigns it): for every
    non-skipped KV block J at level l, the level-l pooled tokens of J.

    Returns (keys [n, d], values [n, d], bias [n], last_token [n])."""
    ks, vs, bias, last = [], [], [], []
    for J, l in enumerate(mask_row):
        l = int(l)
        if l == SKIP:
            continue
        g = 1 << l
        p0 = (J * block) // g
        p1 = min((J + 1) * block, N) // g
        ks.append(kp[l][b, hk, p0:p1])
        vs.append(vp[l][b, hk, p0:p1])
        bias.append(np.full(p1 - p0, level_bias(l)))
        last.append((np.arange(p0, p1) + 1) * g - 1)
    if not ks:
        d = kp[0].shape[-1]
        return np.zeros((0, d)), np.zeros((0, d)), np.zeros(0), np.zeros(0, dtype=np.int64)
    return np.concatenate(ks), np.concatenate(vs), np.concatenate(bias), np.concatenate(last)


def attention(q, kp, vp, mask, block: int, sm_scale: float, causal: bool,
              rows: Optional[Iterable[Tuple[int, int, int]]] = None, p_e4m3: bool = False):
    """Adaptive pyramid attention ([article] Method; [news] Methodology 4,
    ordinary scaled dot-product attention).  For query token i of block I:

        z_p = sm_scale * q_i . K^l[p] + ln(2^l)     over the key set of I
        o_i = sum_p softmax(z)_p V^l[p],   lse_i = log sum_p exp(z_p)

    with readings R1-R4.  q: [B, Hq, N, d]; kp/vp: lists of the pyramid
    levels (level 0 first) as returned by :func:`build_pyramid`; mask
    [B, Hq, nQB, nKB].  Returns (o [B,Hq,N,d], lse [B,Hq,N]); when ``rows``
    lists (b, h, I) triples only those query blocks are computed (the rest
    stay NaN).  With ``p_e4m3`` the output's numerator uses the e4m3
    probabilities of reading R14 (:func:`softmax_pv_e4m3`)."""
    q = _f64(q)
    mask = np.asarray(mask.cpu() if hasattr(mask, "cpu") else mask).astype(np.int64)
    B, Hq, N, d = q.shape
    Hkv = kp[0].shape[1]
    grp = Hq // Hkv
    nb = -(-N // block)
    o = np.full((B, Hq, N, d), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nb)]
    for b, h, I in rows:
        i0, i1 = I * block, min((I + 1) * block, N)
        keys, vals, bias, last = gather_keys(kp, vp, mask[b, h, I], block, N, b, h // grp)
        z = sm_scale * (q[b, h, i0:i1] @ keys.T) + bias[None, :]
        visible = np.ones(z.shape, dtype=bool)
        if causal:
            qi = np.arange(i0, i1)
            visible = last[None, :] <= qi[:, None]
            z = np.where(visible, z, -np.inf)
        empty = ~visible.any(axis=1)
        m = z.max(axis=1, keepdims=True) if z.shape[1] else np.zeros((i1 - i0, 1))
        m = np.where(empty[:, None], 0.0, m)
        e = np.exp(z - m)
        s = e.sum(axis=1)
        if p_e4m3:
            o_rows = softmax_pv_e4m3(z, vals)
        else:
            o_rows = (e @ vals) / np.where(empty, 1.0, s)[:, None]
        o[b, h, i0:i1] = np.where(empty[:, None], 0.0, o_rows)
        lse[b, h, i0:i1] = np.where(empty, -np.inf, m[:, 0] + np.log(np.where(empty, 1.0, s)))
    return o, lse


def attention_backward(q, k, v, mask, block: int, sm_scale: float, causal: bool, levels: int, dout,
                       rows: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Gradients of adaptive pyramid attention with respect to Q, K and V
    (not on the pages' hot path: the news review claims end-to-end
    training, the summary article pairs PSA with distillation).  The mask
    is a fixed selection.  For query i of block I, with P = softmax(z) over
    the key set of I (as in :func:`attention`) and upstream gradient dO_i:

        dV^l[p] += P_ip dO_i,      dP_ip = dO_i . V^l[p],
        D_i = sum_p P_ip dP_ip,    dZ_ip = P_ip (dP_ip - D_i),
        dQ_i = sm_scale sum_p dZ_ip K^l[p],
        dK^l[p] += sm_scale dZ_ip q_i,

    then through the pooling of level l (a mean of 2^l consecutive tokens):
    dK[t] += dK^l[t >> l] / 2^l, and the same for V.  Rows with no visible
    key contribute nothing.  q: [B, Hq, N, d]; k, v: [B, Hkv, N, d];
    dout: [B, Hq, N, d].  Returns (dq, dk, dv) in float64.  When ``rows``
    lists (b, h, I) triples only those query blocks are visited: their dq
    rows are complete (a row's dq depends only on its own key set), dk and
    dv then hold only those blocks' contributions."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    dout = _f64(dout)
    kp, vp = build_pyramid(k, v, levels)
    mask = np.asarray(mask.cpu() if hasattr(mask, "cpu") else mask).astype(np.int64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    nb = -(-N // block)
    dq = np.zeros_like(q)
    dkp = [np.zeros_like(x) for x in kp]
    dvp = [np.zeros_like(x) for x in vp]
    want = None if rows is None else set(rows)
    for b in range(B):
        for h in range(Hq):
            hk = h // grp
            for I in range(nb):
                if want is not None and (b, h, I) not in want:
                    continue
                i0, i1 = I * block, min((I + 1) * block, N)
                # the key set of I, remembering where each key came from
                src = []
                for J, l in enumerate(mask[b, h, I]):
                    l = int(l)
                    if l == SKIP:
                        continue
                    g = 1 << l
                    for pp in range((J * block) // g, min((J + 1) * block, N) // g):
                        src.append((l, pp))
                if not src:
                    continue
                keys = np.stack([kp[l][b, hk, pp] for l, pp in src])
                vals = np.stack([vp[l][b, hk, pp] for l, pp in src])
                bias = np.array([level_bias(l) for l, _ in src])
                last = np.array([(pp + 1) * (1 << l) - 1 for l, pp in src])
                z = sm_scale * (q[b, h, i0:i1] @ keys.T) + bias[None, :]
                if causal:
                    z = np.where(last[None, :] <= np.arange(i0, i1)[:, None], z, -np.inf)
                P = _softmax_rows(z)                                        # [rows, n]
                dO = dout[b, h, i0:i1]
                dP = dO @ vals.T
                D = (P * dP).sum(axis=1, keepdims=True)
                dZ = P * (dP - D)
                dq[b, h, i0:i1] += sm_scale * (dZ @ keys)
                gk = sm_scale * (dZ.T @ q[b, h, i0:i1])                     # [n, d]
                gv = P.T @ dO
                for n_, (l, pp) in enumerate(src):
                    dkp[l][b, hk, pp] += gk[n_]
                    dvp[l][b, hk, pp] += gv[n_]
    return dq, pool_backward(dkp, N), pool_backward(dvp, N)


def pool_backward(grads: List[np.ndarray], N: int) -> np.ndarray:
    """Gradient through the pyramid: level l token t is the mean of input
    tokens t*2^l .. t*2^l + 2^l - 1, so each of them receives 1/2^l of its
    gradient; level 0 is the input itself."""
    out = grads[0].copy()
    for l in range(1, len(grads)):
        g = 1 << l
        out += np.repeat(grads[l], g, axis=2)[:, :, :N] / g
    return out


def executed_flops(mask, N: int, block: int, d: int, causal: bool = False) -> float:
    """Useful work of one attention call: 4 * d * sum over (b, h, I) of
    (valid query rows of I) * (pooled key rows fetched for I).  Diagonal
    blocks count in full under causal masking; tile padding is not work."""
    m = np.asarray(mask.cpu() if hasattr(mask, "cpu") else mask).astype(np.int64)
    B, H, nqb, nkb = m.shape
    qrows = np.array([min((I + 1) * block, N) - I * block for I in range(nqb)], dtype=np.float64)
    total = 0.0
    for l in range(4):
        g = 1 << l
        krows = np.array([(min((J + 1) * block, N) - J * block) // g for J in range(nkb)], dtype=np.float64)
        sel = (m == l)
        total += float((sel * qrows[None, None, :, None] * krows[None, None, None, :]).sum())
    return 4.0 * d * total
