"""Pins for the CPU oracle: each oracle function is checked against
something other than itself.

  function              pins
  --------------------  ---------------------------------------------------------
  pool_level            hand-computed golden values; constant groups are a fixed
                        point; a linear ramp pools to the group midpoints (closed
                        form); direct mean == progressive pairwise pooling
  block_cosine          closed forms (parallel = 1, orthogonal = 0, antipodal =
                        -1, single key = 1); the algebraic identity
                        (|sum u_i|^2 - sum |u_i|^2) / (n(n-1)); scale invariance
  sampling_mass         sum over J == 1; pure-Python brute force; torch.softmax
                        (an independent library routine); one-hot alignment
  antidiag_logits/mass  element-wise brute force; stride 1 reduces to the
                        block-summed full softmax (torch); sum over J == 1;
                        pure-Python brute force of the group -> block
                        aggregation at strides 2 and 4 (causal, ragged, GQA)
  ambiguous_pairs /     hand-derived dyadic goldens (threshold at C_J, at
  ambiguous_pairs_      C_J +- 2 eps and +- eps/2, exact ties, near-ties within
  quantile              and outside relative eps, relative vs absolute eps,
                        cosine at cos_min +- eps); every level flip under a
                        1e-7 relative perturbation lies in the band
  assign_levels_row     hand-computed golden cases; monotone in rank; top = 0
  apply_forced_rules    hand-computed golden cases
  assign_levels_quantile_row
                        hand-computed golden cases; L = 1 with t_0 = k/n keeps
                        exactly numpy's stable top-k; per-level counts n/L
  block_means /         hand-computed golden case (ragged block, causal); torch
  meankey_mass          avg_pool1d + torch.softmax (independent routines); sum
                        over J == 1; token order inside a block and a common
                        shift of every key change nothing
  attention             all-level-0 == torch SDPA (fp64); expanded-KV SDPA
                        equivalence; identical-group invariance; NaN in a
                        skipped block changes nothing; pure-Python brute force
                        over an exhaustive {0,1,2,3,SKIP} mask; empty rows
  e4m3_codes /         hand-derived e4m3 bytes (ties to even, subnormals,
  e4m3_values /        saturation); decode of every byte by the format formula;
  quantize_*_e4m3 /    row and head maxima map to 448, shared level-0 key scale,
  attention_fp8         half-ulp error bound; e4m3-exact inputs give attention
  softmax_pv_e4m3 /    hand-rounded e4m3 probabilities (e4m3_softmax_hand.json);
  attention_fp8(pv)    exact-probability rows equal the softmax; whole-binade
                        shifts change nothing, fractional ones do; identical
                        keys give the bias-weighted mean by direct summation;
                        mutations (rounded normaliser, no rounding, rounding
                        after normalising, reference at the exact maximum)
  attention_backward /  torch autograd through torch avg_pool1d and softmax
  pool_backward         (independent routines), with and without causal
                        masking and GQA; central finite differences; all level
                        0 == torch SDPA autograd; sum of dK over tokens is 0;
                        sum of dV is the sum of dO over rows that see a key
  mutation tests        planted mistakes (bias sign, dropped bias, sum instead of
                        mean, wrong block width, inclusive prefix, transposed
                        antidiagonal, rank off by one, ragged mean over the
                        full block, transposed mean-key logits, pooling
                        gradient without 1/2^l, band edges that keep the
                        block itself / use an absolute eps / flip a sign,
                        rank range off by one, n_vis ignoring causality,
                        antidiagonal key groups summed at the wrong width)
                        each make a pin fail
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
from oracle.psa_oracle import SKIP

RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------------------------
# helpers that do NOT use the oracle's code paths
# --------------------------------------------------------------------------------------

def sdpa64(q, k, v, scale, attn_mask=None):
    """torch's fused SDPA in float64 on the CPU: an independent routine."""
    qt = torch.as_tensor(q, dtype=torch.float64)[None, None]
    kt = torch.as_tensor(k, dtype=torch.float64)[None, None]
    vt = torch.as_tensor(v, dtype=torch.float64)[None, None]
    m = None if attn_mask is None else torch.as_tensor(attn_mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)[0, 0].numpy()


def brute_attention_row(qi, i, K, V, mask_row, block, N, scale, causal):
    """Pure-Python loops: pool each used block on the fly, add ln(2^l),
    exponentiate, normalise."""
    zs, vs = [], []
    d = len(qi)
    for J, l in enumerate(mask_row):
        if l == SKIP:
            continue
        g = 2 ** l
        t = J * block
        while t < min((J + 1) * block, N):
            kk = [sum(K[t + u][c] for u in range(g)) / g for c in range(d)]
            vv = [sum(V[t + u][c] for u in range(g)) / g for c in range(d)]
            if (not causal) or (t + g - 1 <= i):
                zs.append(scale * sum(qi[c] * kk[c] for c in range(d)) + l * math.log(2.0))
                vs.append(vv)
            t += g
    if not zs:
        return [0.0] * d, -math.inf
    m = max(zs)
    e = [math.exp(z - m) for z in zs]
    s = sum(e)
    o = [sum(e[p] * vs[p][c] for p in range(len(e))) / s for c in range(d)]
    return o, m + math.log(s)


def rand(*shape):
    return RNG.standard_normal(shape)


# --------------------------------------------------------------------------------------
# pyramid
# --------------------------------------------------------------------------------------

def pin_pyramid_golden(golden_dir, mod=O):
    g = json.load(open(os.path.join(golden_dir, "pyramid_hand.json")))
    x = np.array(g["tokens"], dtype=np.float64).reshape(1, 1, -1, 1)
    err = 0.0
    for l, want in g["levels"].items():
        got = mod.pool_level(x, int(l))[0, 0, :, 0]
        err = max(err, float(np.abs(got - np.array(want)).max()))
    return err


def test_pyramid_golden(golden_dir):
    assert pin_pyramid_golden(golden_dir) == 0.0


def test_pyramid_constant_groups_fixed_point():
    base = rand(1, 2, 16, 5)
    x = np.repeat(base, 8, axis=2)                # every aligned 8-group is constant
    for l in (1, 2, 3):
        got = O.pool_level(x, l)
        want = np.repeat(base, 8 >> l, axis=2)
        assert np.abs(got - want).max() < 1e-14


def test_pyramid_linear_ramp_midpoints():
    N, a, c = 64, 0.37, -1.5
    t = np.arange(N, dtype=np.float64)
    x = (a * t + c).reshape(1, 1, N, 1) * np.ones((1, 1, 1, 3))
    for l in (1, 2, 3):
        g = 2 ** l
        p = np.arange(N // g)
        want = a * (p * g + (g - 1) / 2.0) + c
        assert np.abs(O.pool_level(x, l)[0, 0, :, 1] - want).max() < 1e-12


def test_pyramid_progressive_equals_direct():
    x = rand(2, 3, 40, 7)
    prev = x
    for l in (1, 2, 3):
        prog = 0.5 * (prev[:, :, 0::2] + prev[:, :, 1::2])
        assert np.abs(prog - O.pool_level(x, l)).max() < 1e-13
        prev = prog


# --------------------------------------------------------------------------------------
# block cosine
# --------------------------------------------------------------------------------------

def test_block_cosine_closed_forms():
    d = 4
    e0, e1 = np.eye(d)[0], np.eye(d)[1]
    k = np.zeros((1, 1, 8, d))
    k[0, 0, 0:4] = [2 * e0, 3 * e0, 0.5 * e0, 7 * e0]     # parallel -> 1
    k[0, 0, 4:6] = [e0, e1]                                # orthogonal -> 0
    k[0, 0, 6:8] = [e1, -4 * e1]                           # antipodal -> -1
    assert abs(O.block_cosine(k[:, :, 0:4], 4)[0, 0, 0] - 1) < 1e-14
    assert abs(O.block_cosine(k[:, :, 4:6], 2)[0, 0, 0] - 0) < 1e-14
    assert abs(O.block_cosine(k[:, :, 6:8], 2)[0, 0, 0] + 1) < 1e-14
    one = rand(1, 1, 1, d)
    assert O.block_cosine(one, 4)[0, 0, 0] == 1.0           # single key (ragged tail)


def test_block_cosine_identity_and_zero_key():
    k = rand(1, 2, 37, 6)
    k[0, 1, 5] = 0.0                                        # a zero key has unit vector 0
    blk = 16
    got = O.block_cosine(k, blk)
    for h in range(2):
        for J in range(3):
            keys = k[0, h, J * blk:min((J + 1) * blk, 37)]
            n = len(keys)
            nrm = np.linalg.norm(keys, axis=1)
            u = np.array([keys[i] / nrm[i] if nrm[i] > 0 else np.zeros(6) for i in range(n)])
            s = u.sum(axis=0)
            want = (s @ s - (u * u).sum()) / (n * (n - 1))
            assert abs(got[0, h, J] - want) < 1e-13


def test_block_cosine_scale_invariant():
    k = rand(1, 1, 32, 5)
    scales = np.abs(rand(1, 1, 32, 1)) + 0.1
    assert np.abs(O.block_cosine(k, 8) - O.block_cosine(k * scales, 8)).max() < 1e-13


# --------------------------------------------------------------------------------------
# sampling score
# --------------------------------------------------------------------------------------

def test_sampling_rows_reading():
    assert O.sampling_rows(0, 64, 1000) == [0, 8, 16, 24, 32, 40, 48, 56]
    assert O.sampling_rows(2, 128, 300) == [256, 272, 288]       # rows >= N dropped
    assert O.sampling_rows(1, 128, 10**6) == [128 + 16 * s for s in range(8)]


@pytest.mark.parametrize("causal", [False, True])
def test_sampling_mass_sums_to_one(causal):
    q, k = rand(1, 4, 200, 8), rand(1, 2, 200, 8)
    m = O.sampling_mass(q, k, 32, 0.35, causal=causal)
    assert np.abs(m.sum(axis=-1) - 1).max() < 1e-12
    if causal:
        nb = m.shape[2]
        for I in range(nb):
            assert np.all(m[:, :, I, I + 1:] == 0)


def test_sampling_mass_bruteforce():
    N, d, blk, scale = 52, 3, 16, 0.7
    q, k = rand(1, 2, N, d), rand(1, 1, N, d)
    got = O.sampling_mass(q, k, blk, scale)
    nb = -(-N // blk)
    for h in range(2):
        for I in range(nb):
            rows = [I * blk + s * (blk // 8) for s in range(8) if I * blk + s * (blk // 8) < N]
            acc = [0.0] * nb
            for i in rows:
                z = [scale * sum(q[0, h, i, c] * k[0, 0, j, c] for c in range(d)) for j in range(N)]
                mx = max(z)
                e = [math.exp(x - mx) for x in z]
                s = sum(e)
                for j in range(N):
                    acc[j // blk] += e[j] / s / len(rows)
            assert np.abs(np.array(acc) - got[0, h, I]).max() < 1e-12


def test_sampling_mass_vs_torch_softmax():
    N, d, blk, scale = 300, 16, 64, 0.25
    q, k = rand(2, 3, N, d), rand(2, 3, N, d)
    got = O.sampling_mass(q, k, blk, scale)
    nb = -(-N // blk)
    for b in range(2):
        for h in range(3):
            P = torch.softmax(torch.tensor(q[b, h]) @ torch.tensor(k[b, h]).T * scale, dim=1).numpy()
            for I in range(nb):
                rows = [r for r in range(I * blk, min(I * blk + blk, N)) if (r - I * blk) % (blk // 8) == 0]
                sums = np.array([P[rows, J * blk:(J + 1) * blk].sum(axis=1).mean() for J in range(nb)])
                assert np.abs(sums - got[b, h, I]).max() < 1e-12


def test_sampling_mass_one_hot():
    N, d, blk = 256, 16, 32
    q = np.zeros((1, 1, N, d))
    k = 0.01 * rand(1, 1, N, d)
    Jstar = 5
    k[0, 0, Jstar * blk:(Jstar + 1) * blk, 0] = 1.0
    q[0, 0, :, 0] = 60.0
    m = O.sampling_mass(q, k, blk, 1.0)
    assert np.all(m[0, 0, :, Jstar] > 1 - 1e-12)
    mask = O.make_mask(m, (0.6, 0.8, 0.9, 0.95), 4, blk, False)
    assert np.all(mask[0, 0, :, Jstar] == 0)
    others = np.delete(mask[0, 0], Jstar, axis=1)
    assert np.all(others == SKIP)


# --------------------------------------------------------------------------------------
# antidiagonal score
# --------------------------------------------------------------------------------------

def test_antidiag_logits_bruteforce():
    N, d, S, scale = 24, 3, 4, 0.9
    qh, kh = rand(N, d), rand(N, d)
    A = O.antidiag_logits(qh, kh, S, scale)
    for a in range(N // S):
        for c in range(N // S):
            acc = 0.0
            for s in range(S):
                i, j = a * S + (S - 1 - s), c * S + s      # bottom-left to top-right of the S x S tile
                acc += sum(qh[i, x] * kh[j, x] for x in range(d))
            assert abs(A[a, c] - scale * acc / S) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_antidiag_stride1_is_block_softmax(causal):
    N, d, blk, scale = 96, 8, 32, 0.4
    q, k = rand(1, 2, N, d), rand(1, 1, N, d)
    got = O.antidiag_mass(q, k, blk, 1, scale, causal)
    for h in range(2):
        Z = torch.tensor(q[0, h]) @ torch.tensor(k[0, 0]).T * scale
        if causal:
            Z = Z.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
        P = torch.softmax(Z, dim=1).numpy()
        for I in range(N // blk):
            want = P[I * blk:(I + 1) * blk].reshape(blk, N // blk, blk).sum(axis=2).mean(axis=0)
            assert np.abs(got[0, h, I] - want).max() < 1e-12


def test_antidiag_mass_sums_to_one():
    q, k = rand(1, 4, 256, 8), rand(1, 2, 256, 8)
    m = O.antidiag_mass(q, k, 64, 8, 0.3, causal=True)
    assert np.abs(m.sum(axis=-1) - 1).max() < 1e-12
    for I in range(4):
        assert np.all(m[:, :, I, I + 1:] == 0)


# --------------------------------------------------------------------------------------
# level assignment and forced rules
# --------------------------------------------------------------------------------------

def test_levels_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "levels_hand.json")))
    for case in g["cases"]:
        got = O.assign_levels_row(case["mass"], case["thresholds"], case["levels"])
        assert list(got) == case["expect"], case
        assert list(O.exclusive_prefix(case["mass"])) == case["prefix"]


def test_levels_monotone_in_rank():
    for _ in range(20):
        m = RNG.dirichlet(np.ones(50) * 0.3)
        lev = O.assign_levels_row(m, (0.6, 0.8, 0.9, 0.95), 4)
        order = sorted(range(50), key=lambda J: (-m[J], J))
        ranked = [255 if lev[J] == SKIP else lev[J] for J in order]
        assert ranked == sorted(ranked)
        assert lev[order[0]] == 0


def test_forced_rules_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "forced_hand.json")))
    for c in g["cases"]:
        cos = None if c["cos"] is None else np.array(c["cos"])
        got = O.apply_forced_rules(np.array(c["levels_in"]), c["I"], c["block"], c["L"], c["causal"],
                                   c["n_dense_prefix"], cos, c["cos_min"])
        assert list(got) == c["expect"], c


# --------------------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------------------

def _pyr(k, v, L):
    return O.build_pyramid(k, v, L)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_level0_is_dense_sdpa(causal):
    B, Hq, Hkv, N, d, blk = 1, 4, 2, 200, 16, 32
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    nb = -(-N // blk)
    mask = np.zeros((B, Hq, nb, nb), dtype=np.uint8)
    kp, vp = _pyr(k, v, 4)
    o, lse = O.attention(q, kp, vp, mask, blk, 0.3, causal)
    for h in range(Hq):
        am = None
        if causal:
            am = torch.tril(torch.ones(N, N, dtype=torch.bool))
        want = sdpa64(q[0, h], k[0, h // 2], v[0, h // 2], 0.3, am)
        assert np.abs(o[0, h] - want).max() < 1e-12
        z = 0.3 * q[0, h] @ k[0, h // 2].T
        if causal:
            z = np.where(np.tril(np.ones((N, N), dtype=bool)), z, -np.inf)
        want_lse = torch.logsumexp(torch.tensor(z), dim=1).numpy()
        assert np.abs(lse[0, h] - want_lse).max() < 1e-12


def test_attention_expanded_kv_equivalence():
    """A level-l pooled token with +ln(2^l) equals that token repeated 2^l
    times inside a plain softmax."""
    B, H, N, d, blk, L = 1, 2, 160, 8, 32, 4
    q, k, v = rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d)
    nb = N // blk
    gen = np.random.default_rng(7)
    mask = gen.choice([0, 1, 2, 3, SKIP], size=(B, H, nb, nb)).astype(np.uint8)
    mask[..., 0] = 2
    kp, vp = _pyr(k, v, L)
    o, _ = O.attention(q, kp, vp, mask, blk, 0.4, False)
    for h in range(H):
        for I in range(nb):
            kt, vt = [], []
            for J in range(nb):
                l = int(mask[0, h, I, J])
                if l == SKIP:
                    continue
                g = 2 ** l
                blockk = k[0, h, J * blk:(J + 1) * blk].reshape(blk // g, g, d).mean(axis=1)
                blockv = v[0, h, J * blk:(J + 1) * blk].reshape(blk // g, g, d).mean(axis=1)
                kt.append(np.repeat(blockk, g, axis=0))
                vt.append(np.repeat(blockv, g, axis=0))
            want = sdpa64(q[0, h, I * blk:(I + 1) * blk], np.concatenate(kt), np.concatenate(vt), 0.4)
            assert np.abs(o[0, h, I * blk:(I + 1) * blk] - want).max() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_attention_identical_groups_equal_dense(causal):
    B, H, d, blk = 1, 2, 8, 32
    base_k, base_v = rand(B, H, 24, d), rand(B, H, 24, d)
    k, v = np.repeat(base_k, 8, axis=2), np.repeat(base_v, 8, axis=2)   # N = 192, 8-groups identical
    N = k.shape[2]
    q = rand(B, H, N, d)
    nb = N // blk
    gen = np.random.default_rng(3)
    mask = gen.integers(0, 4, size=(B, H, nb, nb)).astype(np.uint8)
    if causal:
        # only whole groups in the past are visible under pooling, so compare on a dense
        # reference that masks at 8-group granularity for off-diagonal blocks
        for I in range(nb):
            mask[:, :, I, I] = 0
    kp, vp = _pyr(k, v, 4)
    o, _ = O.attention(q, kp, vp, mask, blk, 0.5, causal)
    for h in range(H):
        am = None
        if causal:
            am = torch.tril(torch.ones(N, N, dtype=torch.bool))
        want = sdpa64(q[0, h], k[0, h], v[0, h], 0.5, am)
        assert np.abs(o[0, h] - want).max() < 1e-12


def test_attention_skip_ignores_nan():
    B, H, N, d, blk = 1, 2, 128, 8, 32
    q, k, v = rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d)
    nb = N // blk
    mask = np.random.default_rng(5).choice([0, 1, 2, 3], size=(B, H, nb, nb)).astype(np.uint8)
    mask[0, :, :2, 2] = SKIP
    kp, vp = _pyr(k, v, 4)
    o1, l1 = O.attention(q, kp, vp, mask, blk, 0.3, False)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 2 * blk:3 * blk] = np.nan
    v2[:, :, 2 * blk:3 * blk] = np.nan
    kp2, vp2 = _pyr(k2, v2, 4)
    o2, l2 = O.attention(q, kp2, vp2, mask, blk, 0.3, False)
    assert np.array_equal(o1[:, :, :2 * blk], o2[:, :, :2 * blk])
    assert np.array_equal(l1[:, :, :2 * blk], l2[:, :, :2 * blk])
    assert np.isnan(o2[:, :, 2 * blk:]).all()


@pytest.mark.parametrize("causal", [False, True])
def test_attention_bruteforce_exhaustive_mask(causal):
    """4x4 block grid; the mask lists every value of {0,1,2,3,SKIP} in every
    row position across the grid (cyclic), N ragged (not a block multiple)."""
    H, d, blk = 2, 4, 16
    N = 56                                    # blocks of 16,16,16,8
    q, k, v = rand(1, H, N, d), rand(1, H, N, d), rand(1, H, N, d)
    vals = [0, 1, 2, 3, SKIP]
    mask = np.zeros((1, H, 4, 4), dtype=np.uint8)
    for h in range(H):
        for I in range(4):
            for J in range(4):
                mask[0, h, I, J] = vals[(I * 4 + J + h) % 5]
    kp, vp = _pyr(k, v, 4)
    o, lse = O.attention(q, kp, vp, mask, blk, 0.45, causal)
    for h in range(H):
        for i in range(N):
            want_o, want_lse = brute_attention_row(list(q[0, h, i]), i, k[0, h].tolist(), v[0, h].tolist(),
                                                   [int(x) for x in mask[0, h, i // blk]], blk, N, 0.45, causal)
            assert np.abs(o[0, h, i] - np.array(want_o)).max() < 1e-12
            if math.isinf(want_lse):
                assert lse[0, h, i] == -math.inf
            else:
                assert abs(lse[0, h, i] - want_lse) < 1e-12


def test_attention_empty_rows():
    q, k, v = rand(1, 1, 64, 4), rand(1, 1, 64, 4), rand(1, 1, 64, 4)
    mask = np.full((1, 1, 2, 2), SKIP, dtype=np.uint8)
    mask[0, 0, 1, 0] = 1
    kp, vp = _pyr(k, v, 2)
    o, lse = O.attention(q, kp, vp, mask, 32, 0.5, False)
    assert np.all(o[0, 0, :32] == 0) and np.all(lse[0, 0, :32] == -np.inf)
    assert np.all(np.isfinite(o[0, 0, 32:]))


def test_executed_flops_counts():
    mask = np.array([[[[0, 1], [SKIP, 3]]]], dtype=np.uint8)
    # N = 48, block 32: q rows 32, 16; k rows level0 32 / level1 16/2=8 ; level3 (16)/8=2
    f = O.executed_flops(mask, 48, 32, 4)
    want = 4 * 4 * (32 * 32 + 32 * 8 + 16 * 2)
    assert f == want


# --------------------------------------------------------------------------------------
# mutation tests: planted mistakes in the oracle must make a pin fail
# --------------------------------------------------------------------------------------

def _run_identical_groups_pin():
    try:
        test_attention_identical_groups_equal_dense(False)
        return True
    except AssertionError:
        return False


def test_mutation_bias_sign(monkeypatch):
    monkeypatch.setattr(O, "level_bias", lambda l: -l * math.log(2.0))
    assert not _run_identical_groups_pin()


def test_mutation_bias_dropped(monkeypatch):
    monkeypatch.setattr(O, "level_bias", lambda l: 0.0)
    assert not _run_identical_groups_pin()


def test_mutation_pool_sum(monkeypatch, golden_dir):
    orig = O.pool_level
    monkeypatch.setattr(O, "pool_level", lambda x, l: orig(x, l) * (1 << l))
    assert pin_pyramid_golden(golden_dir, O) > 0


def test_mutation_block_width(monkeypatch):
    orig = O._block_sum
    monkeypatch.setattr(O, "_block_sum", lambda p, w, n: orig(np.roll(p, 1, axis=1), w, n))
    with pytest.raises(AssertionError):
        test_sampling_mass_bruteforce()


def test_mutation_inclusive_prefix(monkeypatch, golden_dir):
    def bad(mass_row, thresholds, levels):
        mass_row = np.asarray(mass_row, dtype=np.float64)
        order = sorted(range(len(mass_row)), key=lambda J: (-mass_row[J], J))
        out = np.empty(len(mass_row), dtype=np.int64)
        C = 0.0
        for J in order:
            C += mass_row[J]
            lev = sum(1 for t in thresholds if t <= C)
            out[J] = SKIP if lev >= levels else lev
        return out
    monkeypatch.setattr(O, "assign_levels_row", bad)
    with pytest.raises(AssertionError):
        test_levels_golden(golden_dir)


def test_mutation_antidiag_not_reversed(monkeypatch):
    def bad(qh, kh, stride, sm_scale):
        N, d = qh.shape
        G = N // stride
        A = np.zeros((G, G))
        for s in range(stride):
            A += qh[np.arange(G) * stride + s] @ kh[np.arange(G) * stride + s].T
        return (sm_scale / stride) * A
    monkeypatch.setattr(O, "antidiag_logits", bad)
    with pytest.raises(AssertionError):
        test_antidiag_logits_bruteforce()


def test_mutation_transposed_attention_operand(monkeypatch):
    """Swapping K and V in the key gather must break the dense pin."""
    orig = O.gather_keys

    def bad(kp, vp, *a, **kw):
        return orig(vp, kp, *a, **kw)
    monkeypatch.setattr(O, "gather_keys", bad)
    with pytest.raises(AssertionError):
        test_attention_level0_is_dense_sdpa(False)


# --------------------------------------------------------------------------------------
# rank-based (quantile / top-k) levels, reading R10
# --------------------------------------------------------------------------------------

def test_quantile_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "quantile_hand.json")))
    for c in g["cases"]:
        got = O.assign_levels_quantile_row(c["mass"], c["thresholds"], c["levels"], c["n_visible"])
        assert list(got) == c["expect"], (c, list(got))


@pytest.mark.parametrize("n,k", [(16, 5), (32, 1), (8, 8), (64, 40)])
def test_quantile_binary_is_topk(n, k):
    """L = 1 and t_0 = k/n (exact in binary for these n) keep exactly the k
    heaviest blocks: numpy's stable argsort of -mass is the independent
    routine."""
    m = RNG.random(n)
    got = O.assign_levels_quantile_row(m, [k / n], 1, n)
    keep = set(np.argsort(-m, kind="stable")[:k].tolist())
    assert {J for J in range(n) if got[J] == 0} == keep
    assert all(got[J] == SKIP for J in range(n) if J not in keep)


def test_quantile_level_counts_and_monotone():
    n, L = 32, 4
    m = RNG.random(n)
    got = O.assign_levels_quantile_row(m, [0.25, 0.5, 0.75, 1.0], L, n)
    assert [int((got == l).sum()) for l in range(L)] == [8, 8, 8, 8]
    order = np.argsort(-m, kind="stable")
    assert all(got[order[i]] <= got[order[i + 1]] for i in range(n - 1))


# --------------------------------------------------------------------------------------
# mean-key scorer, reading R11
# --------------------------------------------------------------------------------------

def _meankey_golden_case(golden_dir, causal, mod=O):
    g = json.load(open(os.path.join(golden_dir, "meankey_hand.json")))
    q = torch.tensor(g["q"], dtype=torch.float64)[None, None]
    k = torch.tensor(g["k"], dtype=torch.float64)[None, None]
    got = mod.meankey_mass(q, k, g["block"], g["sm_scale"], causal)[0, 0]
    want = np.array(g["expect_causal" if causal else "expect"])
    return np.abs(got - want).max()


@pytest.mark.parametrize("causal", [False, True])
def test_meankey_golden(golden_dir, causal):
    assert _meankey_golden_case(golden_dir, causal) <= 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_meankey_vs_torch(causal):
    """Block means from torch's avg_pool1d (ceil_mode, pad excluded from the
    count), logits and softmax from torch: an independent path."""
    B, Hq, Hkv, N, d, blk = 2, 4, 2, 77, 8, 16
    q = torch.randn(B, Hq, N, d, dtype=torch.float64)
    k = torch.randn(B, Hkv, N, d, dtype=torch.float64)
    def pool(x):
        y = x.reshape(-1, N, d).transpose(1, 2)                     # [*, d, N]
        y = torch.nn.functional.avg_pool1d(y, blk, blk, ceil_mode=True, count_include_pad=False)
        return y.transpose(1, 2).reshape(x.shape[0], x.shape[1], -1, d)
    qm, km = pool(q), pool(k)
    km = km.repeat_interleave(Hq // Hkv, dim=1)
    z = 0.3 * qm @ km.transpose(-1, -2)
    nb = z.shape[-1]
    if causal:
        z = z.masked_fill(torch.ones(nb, nb, dtype=torch.bool).triu(1), float("-inf"))
    want = torch.softmax(z, dim=-1).numpy()
    got = O.meankey_mass(q, k, blk, 0.3, causal)
    assert np.abs(got - want).max() <= 1e-14


def test_meankey_invariants():
    B, H, N, d, blk = 1, 2, 100, 6, 20
    q = torch.randn(B, H, N, d, dtype=torch.float64)
    k = torch.randn(B, H, N, d, dtype=torch.float64)
    base = O.meankey_mass(q, k, blk, 0.5, False)
    assert np.allclose(base.sum(axis=-1), 1.0, atol=1e-14)
    perm = torch.cat([torch.randperm(blk) + J * blk for J in range(N // blk)])
    assert np.abs(O.meankey_mass(q[:, :, perm], k[:, :, perm], blk, 0.5, False) - base).max() <= 1e-13
    shifted = O.meankey_mass(q, k + torch.randn(d, dtype=torch.float64), blk, 0.5, False)
    assert np.abs(shifted - base).max() <= 1e-12
    causal = O.meankey_mass(q, k, blk, 0.5, True)[0, 0]
    assert np.all(causal[np.triu_indices(N // blk, 1)] == 0.0) and causal[0, 0] == 1.0


def test_mutation_quantile_rank_off_by_one(monkeypatch, golden_dir):
    orig = O.assign_levels_quantile_row

    def planted(mass_row, thresholds, levels, n_visible=None):
        n = len(mass_row)
        nv = n if n_visible is None else n_visible
        return orig(mass_row, [t - 1.0 / nv for t in thresholds], levels, nv)   # (r + 1) / n
    monkeypatch.setattr(O, "assign_levels_quantile_row", planted)
    with pytest.raises(AssertionError):
        test_quantile_golden(golden_dir)


def test_mutation_ragged_mean_over_full_block(monkeypatch, golden_dir):
    def planted(x, block):
        x = O._f64(x)
        B, H, N, d = x.shape
        nb = -(-N // block)
        out = np.empty((B, H, nb, d))
        for J in range(nb):
            out[:, :, J] = x[:, :, J * block:min((J + 1) * block, N)].sum(axis=2) / block
        return out
    monkeypatch.setattr(O, "block_means", planted)
    assert _meankey_golden_case(golden_dir, False) > 1e-3


def test_mutation_meankey_transposed(monkeypatch, golden_dir):
    orig = O.block_means

    # transposed logits: score query block J against key block I
    def planted(q, k, block, sm_scale, causal=False, rows=None):
        qm, km = orig(q, block), orig(k, block)
        z = sm_scale * (qm[0, 0] @ km[0, 0].T).T
        if causal:
            z = np.where(np.tril(np.ones_like(z)) > 0, z, -np.inf)
        return O._softmax_rows(z)[None, None]
    monkeypatch.setattr(O, "meankey_mass", planted)
    assert _meankey_golden_case(golden_dir, False) > 1e-3


# --------------------------------------------------------------------------------------
# backward pass (next row of the scope table): dQ, dK, dV through the levels
# --------------------------------------------------------------------------------------

def torch_psa_grads(q, k, v, mask, block, sm_scale, causal, levels, dout):
    """The forward written again with torch ops (avg_pool1d pyramid, gather,
    softmax), differentiated by torch autograd."""
    q = q.clone().requires_grad_(True)
    k = k.clone().requires_grad_(True)
    v = v.clone().requires_grad_(True)
    B, Hq, N, d = q.shape
    grp = Hq // k.shape[1]
    nb = -(-N // block)

    def pool(x, l):
        if l == 0:
            return x
        g = 1 << l
        y = x.reshape(-1, N, d).transpose(1, 2)
        y = torch.nn.functional.avg_pool1d(y, g, g)
        return y.transpose(1, 2).reshape(x.shape[0], x.shape[1], -1, d)
    kl = [pool(k, l) for l in range(levels)]
    vl = [pool(v, l) for l in range(levels)]
    loss = q.new_zeros(())
    for b in range(B):
        for h in range(Hq):
            for I in range(nb):
                i0, i1 = I * block, min((I + 1) * block, N)
                ks, vs, bs, lastt = [], [], [], []
                for J in range(nb):
                    l = int(mask[b, h, I, J])
                    if l == SKIP:
                        continue
                    g = 1 << l
                    p0, p1 = (J * block) // g, min((J + 1) * block, N) // g
                    ks.append(kl[l][b, h // grp, p0:p1])
                    vs.append(vl[l][b, h // grp, p0:p1])
                    bs += [l * math.log(2.0)] * (p1 - p0)
                    lastt += [(p + 1) * g - 1 for p in range(p0, p1)]
                if not ks:
                    continue
                z = sm_scale * q[b, h, i0:i1] @ torch.cat(ks).T + torch.tensor(bs, dtype=q.dtype)
                if causal:
                    vis = torch.tensor(lastt)[None, :] <= torch.arange(i0, i1)[:, None]
                    z = z.masked_fill(~vis, float("-inf"))
                    keep = vis.any(dim=1)
                else:
                    keep = torch.ones(i1 - i0, dtype=torch.bool)
                p_ = torch.softmax(z[keep], dim=-1)
                loss = loss + (p_ @ torch.cat(vs) * dout[b, h, i0:i1][keep]).sum()
    loss.backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def _bwd_case(causal, seed=5):
    g = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, N, d, blk, L = 1, 4, 2, 96, 8, 16, 4
    q = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
    nb = N // blk
    m = torch.randint(0, L + 1, (B, Hq, nb, nb), generator=g)
    m = torch.where(m == L, torch.full_like(m, SKIP), m)
    return q, k, v, m, blk, 0.35, causal, L, do


@pytest.mark.parametrize("causal", [False, True])
def test_backward_vs_torch_autograd(causal):
    args = _bwd_case(causal)
    got = O.attention_backward(*args)
    want = torch_psa_grads(*args)
    for a_, b_ in zip(got, want):
        assert np.abs(a_ - b_).max() <= 1e-12


def test_backward_finite_differences():
    q, k, v, m, blk, sc, causal, L, do = _bwd_case(True, seed=9)
    dq, dk, dv = O.attention_backward(q, k, v, m, blk, sc, causal, L, do)

    def loss(q_, k_, v_):
        kl, vl = O.build_pyramid(k_, v_, L)
        o, _ = O.attention(q_, kl, vl, m, blk, sc, causal)
        return float((np.nan_to_num(o) * do.numpy()).sum())
    eps = 1e-6
    rng = np.random.default_rng(0)
    for which, grad, t in (("q", dq, q), ("k", dk, k), ("v", dv, v)):
        for _ in range(4):
            idx = tuple(int(rng.integers(n)) for n in t.shape)
            tp, tm = t.clone(), t.clone()
            tp[idx] += eps
            tm[idx] -= eps
            args_p = {"q": (tp, k, v), "k": (q, tp, v), "v": (q, k, tp)}[which]
            args_m = {"q": (tm, k, v), "k": (q, tm, v), "v": (q, k, tm)}[which]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def test_backward_level0_is_dense_sdpa():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 1, 48, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, 48, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, 48, 8, generator=g, dtype=torch.float64)
    do = torch.randn(1, 1, 48, 8, generator=g, dtype=torch.float64)
    mask = torch.zeros(1, 1, 3, 3, dtype=torch.int64)
    dq, dk, dv = O.attention_backward(q, k, v, mask, 16, 0.4, False, 4, do)
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=0.4)
    (o * do).sum().backward()
    for a_, b_ in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        assert np.abs(a_ - b_.numpy()).max() <= 1e-12


def test_backward_sum_invariants():
    q, k, v, m, blk, sc, causal, L, do = _bwd_case(True, seed=11)
    dq, dk, dv = O.attention_backward(q, k, v, m, blk, sc, causal, L, do)
    kl, vl = O.build_pyramid(k, v, L)
    _, lse = O.attention(q, kl, vl, m, blk, sc, causal)
    seen = np.isfinite(lse)                                    # rows with a visible key
    assert np.abs(dk.sum(axis=2)).max() <= 1e-12
    grp = q.shape[1] // k.shape[1]
    want = (do.numpy() * seen[..., None]).reshape(1, k.shape[1], grp, -1, q.shape[-1]).sum(axis=(2, 3))
    assert np.abs(dv.sum(axis=2) - want).max() <= 1e-12


def test_mutation_pool_backward_without_scale(monkeypatch):
    def planted(grads, N):
        out = grads[0].copy()
        for l in range(1, len(grads)):
            out += np.repeat(grads[l], 1 << l, axis=2)[:, :, :N]
        return out
    monkeypatch.setattr(O, "pool_backward", planted)
    with pytest.raises(AssertionError):
        test_backward_vs_torch_autograd(False)


# --------------------------------------------------------------------------------------
# the parity band: ambiguous_pairs / ambiguous_pairs_quantile
# --------------------------------------------------------------------------------------

def _row(mass):
    return np.asarray(mass, dtype=np.float64)[None, None, None, :]


def pin_ambiguous_golden(golden_dir, mod=O):
    """Number of hand-derived band cases the oracle gets wrong (0 = pinned)."""
    g = json.load(open(os.path.join(golden_dir, "ambiguous_hand.json")))
    eps = g["eps"]
    wrong = 0
    for case in g["mass_cases"]:
        got = mod.ambiguous_pairs(_row(case["mass"]), case["thresholds"], eps)[0, 0, 0]
        wrong += int(got.tolist() != case["expect"])
    c = g["cos_case"]
    cos = np.asarray(c["blockcos"], dtype=np.float64)[None, None, :]
    got = mod.ambiguous_pairs(_row(c["mass"]), c["thresholds"], eps, blockcos=cos, cos_min=c["cos_min"])[0, 0, 0]
    wrong += int(got.tolist() != c["expect"])
    off = mod.ambiguous_pairs(_row(c["mass"]), c["thresholds"], eps, blockcos=cos, cos_min=-3.0)[0, 0, 0]
    wrong += int(off.any())
    for case in g["quantile_cases"]:
        n = len(case["mass"])
        mass = np.zeros((1, 1, n, n))
        mass[0, 0, case["I"]] = case["mass"]
        got = mod.ambiguous_pairs_quantile(mass, case["thresholds"], len(case["thresholds"]), case["causal"], eps,
                                           rows=[(0, 0, case["I"])])[0, 0, case["I"]]
        wrong += int(got.tolist() != case["expect"])
    return wrong


def test_ambiguous_golden(golden_dir):
    assert pin_ambiguous_golden(golden_dir) == 0


def test_ambiguous_band_brackets_every_fp32_flip():
    """Every pair whose level changes when the masses are perturbed by a
    relative 1e-7 (the size of fp32 rounding of an fp64 mass) must lie in
    the band.  The rows are random, with a planted near-tie and thresholds
    placed on (or within 5e-7 of) exact prefixes so that flips do happen;
    the band stays a small fraction of the pairs."""
    rng = np.random.default_rng(7)
    flips = flagged = total = 0
    for _ in range(200):
        n = int(rng.integers(6, 40))
        m = rng.dirichlet(np.ones(n))
        m[rng.integers(0, n)] = m[rng.integers(0, n)] * (1 + 3e-8)        # plant a near-tie
        m = m / m.sum()
        C = np.sort(O.exclusive_prefix(m))
        k1, k2, k3 = rng.choice(np.arange(1, n), size=3, replace=False)
        th = tuple(sorted((C[k1], C[k2] + 5e-7, C[k3] + 3e-6, 2.0)))
        amb = O.ambiguous_pairs(m[None, None, None, :], th, 1e-6)[0, 0, 0]
        base = O.assign_levels_row(m, th, 4)
        for _ in range(20):
            p = m * (1 + 1e-7 * rng.standard_normal(n))
            moved = O.assign_levels_row(p, th, 4) != base
            flips += int(moved.sum())
            assert not np.any(moved & ~amb)
        flagged += int(amb.sum())
        total += n
    assert flips > 100, flips
    assert flagged <= 0.25 * total, (flagged, total)


def _bad_ambiguous(variant):
    """ambiguous_pairs with one planted mistake (mutation tests)."""
    def bad(mass, thresholds, eps=1e-6, rows=None, blockcos=None, cos_min=-3.0, hq_per_kv=1):
        B, Hq, nqb, nkb = mass.shape
        amb = np.zeros(mass.shape, dtype=bool)
        if rows is None:
            rows = [(b, h, I) for b in range(B) for h in range(Hq) for I in range(nqb)]
        for b, h, I in rows:
            m = mass[b, h, I]
            for J in range(nkb):
                if variant == "absolute_eps":
                    lo = m[m > m[J] + eps].sum()
                    hi = m[m >= m[J] - eps].sum() - m[J]
                else:
                    lo = m[m > m[J] * (1 + eps)].sum()
                    hi = m[m >= m[J] * (1 - eps)].sum() - (0.0 if variant == "hi_keeps_self" else m[J])
                lo_edge = lo + eps if variant == "lo_sign" else lo - eps
                for t in thresholds:
                    if lo_edge <= t <= hi + eps:
                        amb[b, h, I, J] = True
                if blockcos is not None and cos_min > -2.0 and abs(blockcos[b, h // hq_per_kv, J] - cos_min) <= eps:
                    amb[b, h, I, J] = True
        return amb
    return bad


@pytest.mark.parametrize("variant", ["hi_keeps_self", "absolute_eps", "lo_sign"])
def test_mutation_ambiguous_band(monkeypatch, golden_dir, variant):
    monkeypatch.setattr(O, "ambiguous_pairs", _bad_ambiguous(variant))
    assert pin_ambiguous_golden(golden_dir, O) > 0


def test_mutation_ambiguous_quantile_rank_range(monkeypatch, golden_dir):
    """r_hi counted without excluding the block itself widens every rank
    range by one and flags isolated blocks next to a level boundary."""
    def bad(mass, thresholds, levels, causal, eps=1e-6, rows=None):
        B, Hq, nqb, nkb = mass.shape
        amb = np.zeros(mass.shape, dtype=bool)
        for b, h, I in rows:
            m = mass[b, h, I]
            nv = min(I + 1, nkb) if causal else nkb
            for J in range(nkb):
                r_lo = int((m > m[J] * (1 + eps)).sum())
                r_hi = int((m >= m[J] * (1 - eps)).sum())
                lev = {sum(1 for t in thresholds if t <= r / nv) for r in (r_lo, r_hi)}
                amb[b, h, I, J] = len(lev) > 1
        return amb
    monkeypatch.setattr(O, "ambiguous_pairs_quantile", bad)
    assert pin_ambiguous_golden(golden_dir, O) > 0


def test_mutation_ambiguous_quantile_ignores_causal(monkeypatch, golden_dir):
    orig = O.ambiguous_pairs_quantile
    monkeypatch.setattr(O, "ambiguous_pairs_quantile",
                        lambda mass, th, levels, causal, eps=1e-6, rows=None: orig(mass, th, levels, False, eps, rows))
    assert pin_ambiguous_golden(golden_dir, O) > 0


# --------------------------------------------------------------------------------------
# antidiagonal block masses at stride S > 1: pure-Python brute force
# --------------------------------------------------------------------------------------

def brute_antidiag_mass(q, k, block, S, scale, causal):
    """Reading R6 with loops only: the antidiagonal logit of every (query
    group a, key group c), a softmax over the visible key groups, each
    group probability added to the key block holding the group's tokens,
    and the mean over the query groups of each query block."""
    N, d = len(q), len(q[0])
    G = N // S
    nb = -(-N // block)
    mass = [[0.0] * nb for _ in range(nb)]
    groups_in = [0] * nb
    for a in range(G):
        z = {}
        for c in range(G):
            if causal and c > a:
                continue
            acc = 0.0
            for s in range(S):
                i, j = a * S + S - 1 - s, c * S + s
                acc += sum(q[i][x] * k[j][x] for x in range(d))
            z[c] = scale * acc / S
        mx = max(z.values())
        e = {c: math.exp(v - mx) for c, v in z.items()}
        tot = sum(e.values())
        I = (a * S) // block
        groups_in[I] += 1
        for c, v in e.items():
            mass[I][(c * S) // block] += v / tot
    return [[x / groups_in[I] for x in row] for I, row in enumerate(mass)]


@pytest.mark.parametrize("S,causal", [(2, False), (2, True), (4, True), (4, False)])
def test_antidiag_mass_bruteforce_strided(S, causal):
    """N = 40 tokens, block 16 (a ragged last block of 8 tokens), block / S
    = 8 or 4 groups per block, GQA 2:1."""
    N, d, blk, scale = 40, 3, 16, 0.8
    q, k = rand(1, 2, N, d), rand(1, 1, N, d)
    got = O.antidiag_mass(q, k, blk, S, scale, causal)
    for h in range(2):
        want = np.array(brute_antidiag_mass(q[0, h].tolist(), k[0, 0].tolist(), blk, S, scale, causal))
        assert np.abs(got[0, h] - want).max() < 1e-12


def test_mutation_antidiag_group_width(monkeypatch):
    """Summing key groups in runs of the wrong width (tokens per block
    instead of groups per block, here twice the groups) must fail the
    strided brute force, although the masses still sum to one."""
    orig = O._block_sum
    monkeypatch.setattr(O, "_block_sum", lambda p, w, n: orig(p, 2 * w, n))
    q, k = rand(1, 1, 256, 8), rand(1, 1, 256, 8)
    m = O.antidiag_mass(q, k, 64, 8, 0.3, causal=True)
    assert np.abs(m.sum(axis=-1) - 1).max() < 1e-12          # the invariant alone cannot see it
    with pytest.raises(AssertionError):
        test_antidiag_mass_bruteforce_strided(4, True)


# --------------------------------------------------------------------------------------
# FP8 (e4m3) operands, reading R13
# --------------------------------------------------------------------------------------

def pin_e4m3_golden(golden_dir, mod=O):
    g = json.load(open(os.path.join(golden_dir, "e4m3_hand.json")))
    got = mod.e4m3_codes(np.array([c["x"] for c in g["cases"]], dtype=np.float32))
    return int((got.astype(np.int64) != np.array([c["code"] for c in g["cases"]])).sum())


def test_e4m3_golden(golden_dir):
    assert pin_e4m3_golden(golden_dir) == 0


def test_e4m3_values_decode_by_formula():
    """Every byte but the two NaN codes decodes to the value the format
    definition gives (pure-Python decode)."""
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    got = O.e4m3_values(codes)
    for c, v in zip(codes.tolist(), got.tolist()):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        want = (2.0 ** -6) * m / 8 if e == 0 else 2.0 ** (e - 7) * (1 + m / 8)
        assert v == (-want if s else want), (c, v, want)


def test_quantize_rows_e4m3_properties():
    x = rand(2, 3, 40, 16).astype(np.float32)
    x[0, 0, 5] = 0.0                                   # an all-zero row
    codes, scale = O.quantize_rows_e4m3(x)
    vals = O.e4m3_values(codes)
    assert np.all(codes[0, 0, 5] == 0) and scale[0, 0, 5] == 0
    am = np.abs(x).max(axis=-1)
    nz = am > 0
    # each row's largest magnitude maps to +-448 exactly
    assert np.all(np.abs(vals).max(axis=-1)[nz] == 448.0)
    np.testing.assert_array_equal(scale, (am / np.float32(448)).astype(np.float32))
    # relative error of every normal-range element: at most half an e4m3 ulp (2^-4)
    y = x * (np.float32(448) / np.where(nz, am, 1))[..., None]
    normal = np.abs(y) >= 2.0 ** -6
    assert np.all(np.abs(vals - y)[normal] <= 2.0 ** -4 * np.abs(y)[normal] + 1e-6)


def test_quantize_heads_e4m3_shares_level0_scale():
    k = rand(1, 2, 64, 8).astype(np.float32)
    kl, _ = O.build_pyramid(k, k, 4)
    codes, scale = O.quantize_heads_e4m3(kl)
    am = np.abs(k).reshape(1, 2, -1).max(axis=-1)
    np.testing.assert_array_equal(scale, (am / np.float32(448)).astype(np.float32))
    for lv in range(4):
        vals = O.e4m3_values(codes[lv])
        assert np.abs(vals).max() <= 448.0
    assert np.abs(O.e4m3_values(codes[0])).reshape(1, 2, -1).max(axis=-1).tolist() == [[448.0, 448.0]]


def test_attention_fp8_exact_inputs_equal_attention():
    """Inputs whose scaled values are already e4m3 numbers (every row and
    head has an element of magnitude 448, all values on the e4m3 grid, so
    the scale is 1) give exactly the plain attention."""
    rng = np.random.default_rng(3)
    grid = O.e4m3_values(np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8))
    grid = grid[np.abs(grid) <= 64]
    N, d, blk = 64, 8, 16
    q = rng.choice(grid, size=(1, 1, N, d))
    k = rng.choice(grid, size=(1, 1, N, d))
    q[..., 0] = 448.0
    k[0, 0, 0, 0] = 448.0
    v = rng.standard_normal((1, 1, N, d))
    mask = np.zeros((1, 1, N // blk, N // blk), dtype=np.uint8)
    scale = 1.0 / 448.0 / 8.0
    o8, l8 = O.attention_fp8(q, [k], [v], mask, blk, scale, False)
    o, l = O.attention(q, [k], [v], mask, blk, scale, False)
    np.testing.assert_array_equal(o8, o)
    np.testing.assert_array_equal(l8, l)


def test_mutation_e4m3_ties_away(monkeypatch, golden_dir):
    """Rounding ties away from zero instead of to even fails the golden."""
    def bad(x32):
        x = np.clip(np.asarray(x32, dtype=np.float64), -448, 448)
        grid = O.e4m3_values(np.arange(256, dtype=np.uint8))
        out = []
        for v in x.ravel():
            dist = np.abs(grid - v)
            dist[np.isnan(dist)] = np.inf
            best = np.flatnonzero(dist == dist.min())
            out.append(max(best, key=lambda c: abs(grid[c])))
        return np.array(out, dtype=np.uint8).reshape(x.shape)
    monkeypatch.setattr(O, "e4m3_codes", bad)
    assert pin_e4m3_golden(golden_dir, O) > 0


def test_mutation_head_scale_per_level(monkeypatch):
    """A key scale taken per level instead of from level 0 breaks the
    shared-scale property."""
    orig = O.quantize_heads_e4m3

    def bad(levels):
        out = [orig([x]) for x in levels]
        return [c[0][0] for c in out], out[-1][1]
    monkeypatch.setattr(O, "quantize_heads_e4m3", bad)
    with pytest.raises(AssertionError):
        test_quantize_heads_e4m3_shares_level0_scale()


# ======================================================================================
# FP8 probabilities and values, reading R14
# ======================================================================================

def pin_softmax_pv_golden(golden_dir, mod=O):
    """Largest deviation of softmax_pv_e4m3 from the hand-rounded rows."""
    g = json.load(open(os.path.join(golden_dir, "e4m3_softmax_hand.json")))
    worst = 0.0
    for r in g["rows"]:
        a = np.array(r["logits_log2"])
        v = np.array(r["values"])[:, None]
        den = np.sum(np.exp2(a - r["reference"]).astype(np.float32).astype(np.float64))   # P in fp32
        want = float(np.dot(r["p_e4m3"], v[:, 0]) / den)
        got = float(mod.softmax_pv_e4m3((a * np.log(2.0))[None, :], v)[0, 0])
        worst = max(worst, abs(got - want) / abs(want))
    return worst


def test_softmax_pv_e4m3_golden(golden_dir):
    assert pin_softmax_pv_golden(golden_dir) < 1e-14


def test_softmax_pv_e4m3_exact_probabilities_equal_softmax():
    """Logits a whole number of binades apart, all within 6 of the largest,
    give probabilities that e4m3 holds exactly: the result is the plain
    softmax times V."""
    rng = np.random.default_rng(11)
    a = rng.integers(-6, 1, size=(5, 9)).astype(np.float64) + 2.0
    a[:, 0] = 2.0
    v = rng.standard_normal((9, 3))
    z = a * np.log(2.0)
    e = np.exp(z - z.max(axis=1, keepdims=True))
    want = (e @ v) / e.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(O.softmax_pv_e4m3(z, v), want, rtol=1e-13, atol=0)


def test_softmax_pv_e4m3_binade_shifts():
    """Moving every logit of a row by a whole number of binades changes
    nothing while the probabilities stay in e4m3's normal range; a shift by
    a fraction of a binade moves the rounding grid and changes the result."""
    rng = np.random.default_rng(12)
    a = rng.uniform(-4.5, 0.0, size=(6, 20))
    v = rng.standard_normal((20, 4))
    base = O.softmax_pv_e4m3(a * np.log(2.0), v)
    for k in (-3, 1, 7):
        np.testing.assert_array_equal(O.softmax_pv_e4m3((a + k) * np.log(2.0), v), base)
    assert np.abs(O.softmax_pv_e4m3((a + 0.37) * np.log(2.0), v) - base).max() > 1e-4


def test_attention_fp8_pv_uniform_keys_closed_form():
    """Zero queries make every logit its level bias (a whole number of
    binades), so the probabilities are powers of two (exact in e4m3);
    values on the e4m3
    grid with a largest magnitude of 448 keep a scale of 1, and pairs of
    equal tokens pool to themselves.  The output is then the bias-weighted
    mean of the values of the key set, by direct summation."""
    rng = np.random.default_rng(13)
    N, d, blk, L = 64, 4, 16, 2
    grid = O.e4m3_values(np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8))
    grid = grid[np.abs(grid) <= 64]
    q = np.zeros((1, 1, N, d))
    k = rng.standard_normal((1, 1, N, d))
    vh = rng.choice(grid, size=(1, 1, N // 2, d))
    vh[0, 0, 0, 0] = 448.0
    v = np.repeat(vh, 2, axis=2)
    kl, vl = O.build_pyramid(k, v, L)
    mask = np.array([[[[0, 1, SKIP, 1], [1, 0, 1, SKIP], [SKIP, SKIP, 0, 0], [1, 1, 1, 1]]]], dtype=np.uint8)
    o, _ = O.attention_fp8(q, kl, vl, mask, blk, 0.3, False, pv=True)
    for I in range(N // blk):
        wts, vals = [], []
        for J, lv in enumerate(mask[0, 0, I]):
            if lv == SKIP:
                continue
            g = 1 << int(lv)
            for p in range(J * blk // g, (J + 1) * blk // g):
                wts.append(2.0 ** int(lv))
                vals.append(vl[int(lv)][0, 0, p])
        want = np.sum(np.array(wts)[:, None] * np.array(vals), axis=0) / np.sum(wts)
        np.testing.assert_allclose(o[0, 0, I * blk:(I + 1) * blk], np.tile(want, (blk, 1)), rtol=1e-13, atol=1e-12)


def _bad_softmax_pv(kind):
    def bad(z, vals):
        a = np.asarray(z, dtype=np.float64) / np.log(2.0)
        amax = a.max(axis=1, keepdims=True)
        M = amax if kind == "exact_max" else np.ceil(amax)
        p = np.exp2(a - M).astype(np.float32)
        pq = O.e4m3_values(O.e4m3_codes(p))
        den = p.astype(np.float64).sum(axis=1, keepdims=True)
        if kind == "rounded_sum":
            return (pq @ vals) / pq.sum(axis=1, keepdims=True)
        if kind == "no_rounding":
            return (p.astype(np.float64) @ vals) / den
        if kind == "round_after_normalising":
            pn = O.e4m3_values(O.e4m3_codes((p / den).astype(np.float32)))
            return pn @ vals
        return (pq @ vals) / den
    return bad


@pytest.mark.parametrize("kind", ["rounded_sum", "no_rounding", "round_after_normalising", "exact_max"])
def test_mutation_softmax_pv(monkeypatch, golden_dir, kind):
    """Normalising by the rounded sum, not rounding, rounding the
    normalised probabilities, or a reference at the exact (not whole-binade)
    maximum each fail the hand-rounded golden."""
    monkeypatch.setattr(O, "softmax_pv_e4m3", _bad_softmax_pv(kind))
    assert pin_softmax_pv_golden(golden_dir, O) > 1e-3


def test_backward_rows_filter_matches_full():
    """Visiting only some query blocks leaves their dq rows exactly as the
    full computation gives them (a row's gradient depends on its own key
    set only)."""
    q, k, v, mask, blk, scale, causal, L, dout = _bwd_case(True)
    full = O.attention_backward(q, k, v, mask, blk, scale, causal, L, dout)
    rows = [(0, 1, 0), (0, 2, 2), (0, 0, 3)]
    part = O.attention_backward(q, k, v, mask, blk, scale, causal, L, dout, rows=rows)
    for b, h, I in rows:
        np.testing.assert_array_equal(part[0][b, h, I * blk:(I + 1) * blk], full[0][b, h, I * blk:(I + 1) * blk])
    assert np.all(part[0][0, 1, blk:2 * blk] == 0)
