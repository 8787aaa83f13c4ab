"""Parity of the mask-policy variants and the mean-key scorer (CUDA path
through the C ABI) with the oracle.

  * mean-key scorer (PSA_MASK_MEANKEY): block masses relative 1e-4 where the
    mass is above 1e-6; masks bit-exact outside the ambiguity band.
  * rank policy (PSA_POLICY_QUANTILE): masks bit-exact except blocks whose
    rank can move across a level boundary between near-equal masses
    (relative 1e-6).  Thresholds are values exact in binary, so both sides
    compare r / n_visible with the same numbers.
  * binary masks: one level (L = 1) through the same generator and kernel.
Attention on top of each mask is checked like the main pipeline (max-abs
2e-2, mean-abs 2e-3 against the oracle in fp64)."""
import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import video_transformers_b200 as P
import workloads as W
from amb_report import check_band
from psa_run import SKIP, attn_errors, levels_of, params_for, run_attention, run_mask, run_pyramid, shape_for

pytestmark = pytest.mark.gpu
DEV = "cuda"


def oracle_mass(w, q, k, rows=None):
    if w.mask_mode == "meankey":
        return O.meankey_mass(q, k, w.block, w.sm_scale, w.causal, rows=rows)
    if w.mask_mode == "sample":
        return O.sampling_mass(q, k, w.block, w.sm_scale, w.causal, rows=rows)
    return O.antidiag_mass(q, k, w.block, w.stride, w.sm_scale, w.causal, rows=rows)


def check_variant(w, q, k, policy):
    shape = shape_for(w)
    mask, mass = run_mask(shape, params_for(w, policy), q, k)
    mask, mass = mask.cpu().numpy(), mass.cpu().numpy().astype(np.float64)
    om = oracle_mass(w, q, k)
    th = [float(np.float32(t)) for t in w.thresholds]
    pol = "quantile" if policy == P.PSA_POLICY_QUANTILE else "mass"
    omask = O.make_mask(om, th, w.levels, w.block, w.causal, w.n_dense_prefix, None, -3.0, w.Hq // w.Hkv,
                        policy=pol)
    if pol == "quantile":
        amb = O.ambiguous_pairs_quantile(om, th, w.levels, w.causal, 1e-6)
    else:
        amb = O.ambiguous_pairs(om, th, 1e-6)
    big = om > 1e-6
    rel = np.abs(mass[big] - om[big]) / om[big]
    assert rel.max() <= 1e-4, rel.max()
    bad = ~amb & (mask != omask)
    assert bad.sum() == 0, "mask mismatches outside the ambiguity band: %d (ambiguous %d)" % (bad.sum(), amb.sum())
    check_band("%s %s/%s L=%d N=%d" % (w.name, w.mask_mode, pol, w.levels, w.N), int(amb.sum()), int(amb.size))
    return mask


@pytest.mark.parametrize("name,grid,heads,causal,block", [
    ("wan14b", (4, 12, 16), (2, 2), False, 128),        # N = 768
    ("wan14b", (3, 9, 16), (4, 2), True, 128),          # N = 432, ragged, GQA, causal
    ("wan1.3b", (3, 10, 12), (2, 2), False, 64),        # N = 360, ragged
    ("qwen2.5vl", (6, 8, 16), (7, 1), True, 128),       # N = 768, GQA 7:1
])
def test_meankey_mask_parity(name, grid, heads, causal, block):
    w = W.reduced(name, grid=grid, heads=heads).replace(mask_mode="meankey", causal=causal, block=block,
                                                        cos_min=-3.0)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    check_variant(w, q.to(DEV), k.to(DEV), P.PSA_POLICY_MASS)


def test_meankey_fp32_inputs():
    w = W.PRESETS["tiny"].replace(mask_mode="meankey", thresholds=(0.5, 0.7, 0.85, 0.9))
    q, k, v, _ = W.make_qkv(w, device="cpu")
    check_variant(w, q.to(DEV), k.to(DEV), P.PSA_POLICY_MASS)


@pytest.mark.parametrize("mode", ["sample", "meankey"])
@pytest.mark.parametrize("causal", [False, True])
def test_quantile_policy_parity(mode, causal):
    w = W.reduced("wan14b", grid=(4, 12, 16), heads=(2, 2)).replace(
        mask_mode=mode, causal=causal, thresholds=(0.25, 0.5, 0.75, 0.875), cos_min=-3.0)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    mask = check_variant(w, q.to(DEV), k.to(DEV), P.PSA_POLICY_QUANTILE)
    if not causal:
        # each level holds (close to) its share of the six blocks of a row
        nb = mask.shape[-1]
        assert np.all((mask == 0).sum(axis=-1) >= nb // 4)


@pytest.mark.parametrize("mode,policy", [("sample", P.PSA_POLICY_MASS), ("meankey", P.PSA_POLICY_QUANTILE)])
def test_binary_mask_one_level(mode, policy):
    """L = 1: the generator emits only {0, SKIP}; with the rank policy and
    t_0 = 3/8 a non-causal row keeps exactly its 3 heaviest of 8 blocks."""
    w = W.reduced("wan14b", grid=(4, 16, 16), heads=(2, 2)).replace(
        mask_mode=mode, levels=1, thresholds=(0.375,), cos_min=-3.0)       # N = 1024, 8 blocks
    q, k, v, _ = W.make_qkv(w, device="cpu")
    mask = check_variant(w, q.to(DEV), k.to(DEV), policy)
    assert set(np.unique(mask).tolist()) <= {0, SKIP}
    if policy == P.PSA_POLICY_QUANTILE:
        assert np.all((mask == 0).sum(axis=-1) == 3)


@pytest.mark.parametrize("mode,policy,levels", [
    ("meankey", P.PSA_POLICY_MASS, 4),
    ("meankey", P.PSA_POLICY_QUANTILE, 4),
    ("sample", P.PSA_POLICY_MASS, 1),
])
def test_attention_on_variant_masks(mode, policy, levels):
    th = (0.6, 0.8, 0.9, 0.95) if policy == P.PSA_POLICY_MASS else (0.25, 0.5, 0.75, 0.875)
    w = W.reduced("wan14b", grid=(3, 9, 16), heads=(2, 2)).replace(
        mask_mode=mode, levels=levels, thresholds=th[:levels], cos_min=-3.0)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    mask, _ = run_mask(shape, params_for(w, policy), q, k)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    kl = levels_of(shape, kp, k) if levels > 1 else [k.double().cpu().numpy()]
    vl = levels_of(shape, vp, v) if levels > 1 else [v.double().cpu().numpy()]
    o, l = O.attention(q, kl, vl, mask.cpu(), w.block, w.sm_scale, w.causal)
    mx, mean, _ = attn_errors(out, o)
    assert mx <= 2e-2 and mean <= 2e-3, (mx, mean)


def test_meankey_quantile_text_prefix_causal_fp32():
    """Every forced rule on top of the new scorer and policy: a text prefix
    (its blocks stay level 0), causal masking (J > I skipped, J == I level
    0), fp32 inputs, GQA 2:1 and a ragged last block."""
    w = W.reduced("cogvideox5b", grid=(3, 10, 15), heads=(4, 2), n_text=30).replace(
        mask_mode="meankey", causal=True, dtype="fp32", thresholds=(0.25, 0.5, 0.75, 0.875), cos_min=-3.0)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    mask = check_variant(w, q.to(DEV), k.to(DEV), P.PSA_POLICY_QUANTILE)
    nb = mask.shape[-1]
    iu = np.triu_indices(nb, 1)
    assert np.all(mask[..., iu[0], iu[1]] == SKIP)
    assert np.all(mask[..., np.arange(nb), np.arange(nb)] == 0)
    assert np.all(mask[..., 0, 0] == 0) and np.all(mask[..., :, 0] == 0)     # block 0 holds text
