"""Full-size parity: each workload preset at its real shape, run the way the
benchmark runs it (inputs generated on the GPU, the whole path through the
C ABI, the persistent kernels at full grid), checked on sampled query
blocks that the oracle recomputes one by one: the mask rows (bit-exact
outside the ambiguity band), the block masses, and the attention rows."""
import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import video_transformers_b200 as P
import workloads as W
from psa_run import SKIP, attn_errors, params_for, run_attention, run_mask, run_pyramid, shape_for

pytestmark = pytest.mark.gpu
DEV = "cuda"


def sample_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    hs = rng.integers(0, w.Hq, size=n)
    Is = rng.integers(0, w.nqb, size=n)
    Is[0], Is[-1] = 0, w.nqb - 1            # first and (ragged) last query block
    return [(0, int(h), int(I)) for h, I in zip(hs, Is)]


@pytest.mark.parametrize("name", ["wan1.3b", "cogvideox5b", "qwen2.5vl", "wan14b"])
def test_fullsize_sampled_parity(name):
    w = W.PRESETS[name]
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    kp, vp, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    mask, mass = run_mask(shape, params_for(w), q, k, bc)
    out, lse, ws = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    torch.cuda.synchronize()
    grp = w.Hq // w.Hkv
    n_amb = n_pairs = 0
    for b, h, I in sample_rows(w, 6, seed=len(name)):
        hk = h // grp
        qh, kh, vh = q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, hk:hk + 1].cpu(), v[b:b + 1, hk:hk + 1].cpu()
        row = [(0, 0, I)]
        if w.mask_mode == "sample":
            om = O.sampling_mass(qh, kh, w.block, w.sm_scale, w.causal, rows=row)
        else:
            om = O.antidiag_mass(qh, kh, w.block, w.stride, w.sm_scale, w.causal, rows=row)
        cos = None
        if bc is not None:
            cos = bc[b:b + 1, hk:hk + 1].cpu().numpy().astype(np.float64)
            ocos = O.block_cosine(kh, w.block)
            assert np.abs(cos - ocos).max() <= 1e-5
        omask = O.make_mask(om, w.thresholds, w.levels, w.block, w.causal, w.n_dense_prefix, cos, w.cos_min,
                            1, rows=row)[0, 0, I]
        amb = O.ambiguous_pairs(om, w.thresholds, 1e-6, row, cos, w.cos_min, 1)[0, 0, I]
        gm = mask[b, h, I].cpu().numpy()
        gmass = mass[b, h, I].cpu().numpy().astype(np.float64)
        big = om[0, 0, I] > 1e-6
        assert (np.abs(gmass[big] - om[0, 0, I][big]) / om[0, 0, I][big]).max() <= 1e-4
        assert np.all((gm == omask) | amb), (name, h, I, int(((gm != omask) & ~amb).sum()))
        n_amb += int(amb.sum())
        n_pairs += amb.size
        # attention rows of this query block, from the GPU pyramid and mask
        kl = [kh.double().numpy()] + [P.pyramid_level(shape, kp, l)[b:b + 1, hk:hk + 1].double().cpu().numpy()
                                      for l in range(1, w.levels)]
        vl = [vh.double().numpy()] + [P.pyramid_level(shape, vp, l)[b:b + 1, hk:hk + 1].double().cpu().numpy()
                                      for l in range(1, w.levels)]
        o, l = O.attention(qh, kl, vl, mask[b:b + 1, h:h + 1].cpu(), w.block, w.sm_scale, w.causal, rows=row)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 2e-2 and mean <= 2e-3, (name, h, I, mx, mean)
    assert P.psa_get_device_status(ws) == P.PSA_OK
    print("%s: %d ambiguous of %d sampled pairs" % (name, n_amb, n_pairs))


@pytest.mark.parametrize("mode,policy", [("meankey", "mass"), ("sample", "quantile")])
def test_fullsize_mask_variants_sampled(mode, policy):
    """The mask variants at the Wan2.1-14B shape, as `bench.py --mask-mode
    meankey` and `--policy quantile` run them: sampled query-block rows of
    the mask (bit-exact outside the ambiguity band) and their masses, then
    the attention rows of those blocks on the GPU mask."""
    w = W.PRESETS["wan14b"].replace(mask_mode=mode, policy=policy)
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    pol = P.PSA_POLICY_QUANTILE if policy == "quantile" else P.PSA_POLICY_MASS
    kp, vp, _ = run_pyramid(shape, k, v)
    mask, mass = run_mask(shape, params_for(w, pol), q, k)
    out, lse, ws = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    torch.cuda.synchronize()
    th = [float(np.float32(t)) for t in w.thresholds]
    for b, h, I in sample_rows(w, 4, seed=7 + len(mode)):
        qh, kh, vh = q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, h:h + 1].cpu(), v[b:b + 1, h:h + 1].cpu()
        row = [(0, 0, I)]
        if mode == "meankey":
            om = O.meankey_mass(qh, kh, w.block, w.sm_scale, w.causal, rows=row)
        else:
            om = O.sampling_mass(qh, kh, w.block, w.sm_scale, w.causal, rows=row)
        omask = O.make_mask(om, th, w.levels, w.block, w.causal, w.n_dense_prefix, None, -3.0, 1, rows=row,
                            policy=policy)[0, 0, I]
        if policy == "quantile":
            amb = O.ambiguous_pairs_quantile(om, th, w.levels, w.causal, 1e-6, rows=row)[0, 0, I]
        else:
            amb = O.ambiguous_pairs(om, th, 1e-6, row)[0, 0, I]
        gm = mask[b, h, I].cpu().numpy()
        gmass = mass[b, h, I].cpu().numpy().astype(np.float64)
        big = om[0, 0, I] > 1e-6
        assert (np.abs(gmass[big] - om[0, 0, I][big]) / om[0, 0, I][big]).max() <= 1e-4
        assert np.all((gm == omask) | amb), (mode, policy, h, I, int(((gm != omask) & ~amb).sum()))
        kl = [kh.double().numpy()] + [P.pyramid_level(shape, kp, l)[b:b + 1, h:h + 1].double().cpu().numpy()
                                      for l in range(1, w.levels)]
        vl = [vh.double().numpy()] + [P.pyramid_level(shape, vp, l)[b:b + 1, h:h + 1].double().cpu().numpy()
                                      for l in range(1, w.levels)]
        o, l = O.attention(qh, kl, vl, mask[b:b + 1, h:h + 1].cpu(), w.block, w.sm_scale, w.causal, rows=row)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 2e-2 and mean <= 2e-3, (mode, policy, h, I, mx, mean)
    assert P.psa_get_device_status(ws) == P.PSA_OK
