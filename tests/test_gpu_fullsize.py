"""Full-size parity: each workload preset at its real shape, run the way the
benchmark runs it (inputs generated on the GPU, the whole path through the
C ABI, the persistent kernels at full grid), checked on sampled query
blocks that the oracle recomputes one by one: the mask rows (bit-exact
outside the ambiguity band), the block masses, and the attention rows.
At least 64 (head, query block) rows per preset: every head of the first,
a middle and the ragged last block, plus random rows."""
import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import video_transformers_b200 as P
import workloads as W
from amb_report import check_band, note
from psa_run import SKIP, attn_errors, params_for, run_attention, run_mask, run_pyramid, shape_for

pytestmark = pytest.mark.gpu
DEV = "cuda"


def sample_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    hs = rng.integers(0, w.Hq, size=n)
    Is = rng.integers(0, w.nqb, size=n)
    Is[0], Is[-1] = 0, w.nqb - 1            # first and (ragged) last query block
    return [(0, int(h), int(I)) for h, I in zip(hs, Is)]


def fullsize_rows(w, n_min=64, seed=0):
    """Every head of the first, a middle and the (ragged) last query block,
    topped up with random (head, block) rows to at least n_min."""
    rows = {(0, h, I) for h in range(w.Hq) for I in (0, w.nqb // 2, w.nqb - 1)}
    rng = np.random.default_rng(seed)
    while len(rows) < n_min:
        rows.add((0, int(rng.integers(0, w.Hq)), int(rng.integers(0, w.nqb))))
    return sorted(rows)


def by_head(rows):
    out = {}
    for b, h, I in rows:
        out.setdefault((b, h), []).append(I)
    return out


def head_levels(shape, base, pyr, b, hk, levels):
    return [base[b:b + 1, hk:hk + 1].double().cpu().numpy()] + \
        [P.pyramid_level(shape, pyr, l)[b:b + 1, hk:hk + 1].double().cpu().numpy() for l in range(1, levels)]


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
    rows = fullsize_rows(w, seed=len(name))
    assert len(rows) >= 64
    n_amb = n_pairs = 0
    cos_cache = {}
    for (b, h), Is in by_head(rows).items():
        hk = h // grp
        qh, kh, vh = q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, hk:hk + 1].cpu(), v[b:b + 1, hk:hk + 1].cpu()
        hrows = [(0, 0, I) for I in Is]
        if w.mask_mode == "sample":
            om = O.sampling_mass(qh, kh, w.block, w.sm_scale, w.causal, rows=hrows)
        else:
            om = O.antidiag_mass(qh, kh, w.block, w.stride, w.sm_scale, w.causal, rows=hrows)
        cos = None
        if bc is not None:
            cos = bc[b:b + 1, hk:hk + 1].cpu().numpy().astype(np.float64)
            if hk not in cos_cache:
                cos_cache[hk] = O.block_cosine(kh, w.block)
                assert np.abs(cos - cos_cache[hk]).max() <= 1e-5
        omask = O.make_mask(om, w.thresholds, w.levels, w.block, w.causal, w.n_dense_prefix, cos, w.cos_min,
                            1, rows=hrows)[0, 0]
        amb = O.ambiguous_pairs(om, w.thresholds, 1e-6, hrows, cos, w.cos_min, 1)[0, 0]
        gm = mask[b, h].cpu().numpy()
        gmass = mass[b, h].cpu().numpy().astype(np.float64)
        for I in Is:
            big = om[0, 0, I] > 1e-6
            assert (np.abs(gmass[I][big] - om[0, 0, I][big]) / om[0, 0, I][big]).max() <= 1e-4
            assert np.all((gm[I] == omask[I]) | amb[I]), (name, h, I, int(((gm[I] != omask[I]) & ~amb[I]).sum()))
            n_amb += int(amb[I].sum())
            n_pairs += amb[I].size
        # attention rows of these query blocks, from the GPU pyramid and mask
        kl = head_levels(shape, k, kp, b, hk, w.levels)
        vl = head_levels(shape, v, vp, b, hk, w.levels)
        o, l = O.attention(qh, kl, vl, mask[b:b + 1, h:h + 1].cpu(), w.block, w.sm_scale, w.causal, rows=hrows)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 2e-2 and mean <= 2e-3, (name, h, Is, mx, mean)
        lg = lse[b, h].cpu().numpy().astype(np.float64)
        sel = ~np.isnan(l[0, 0])
        assert np.abs(lg[sel] - l[0, 0][sel]).max() <= 2e-2
    assert P.psa_get_device_status(ws) == P.PSA_OK
    check_band("%s full size, %d rows" % (name, len(rows)), n_amb, n_pairs)


def test_fullsize_dense_wan14b():
    """The dense reference point the benchmark times: the Wan2.1-14B shape
    with every pair at level 0, checked on sampled query-block rows against
    the oracle's plain softmax attention over all 75,600 keys."""
    w = W.PRESETS["wan14b"]
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    mask = torch.zeros(w.B, w.Hq, w.nqb, w.nqb, dtype=torch.uint8, device=DEV)
    out, lse, ws = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    torch.cuda.synchronize()
    for b, h, I in sample_rows(w, 12, seed=99):
        row = [(0, 0, I)]
        o, l = O.attention(q[b:b + 1, h:h + 1].cpu(), [k[b:b + 1, h:h + 1].cpu().double().numpy()],
                           [v[b:b + 1, h:h + 1].cpu().double().numpy()], mask[b:b + 1, h:h + 1, :, :].cpu(),
                           w.block, w.sm_scale, False, rows=row)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 2e-2 and mean <= 2e-3, (h, I, mx, mean)
    nt, nr = P.psa_attention_plan_stats(shape, ws)
    # every query tile lists all 591 blocks as 128-row segments (the ragged
    # last block included: the plan counts segment rows, not valid tokens)
    assert nr == w.Hq * w.nqb * w.nqb * w.block and nt == w.Hq * w.nqb * w.nqb
    assert P.psa_get_device_status(ws) == P.PSA_OK


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
    n_amb = n_pairs = 0
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
        n_amb += int(amb.sum())
        n_pairs += amb.size
        kl = [kh.double().numpy()] + [P.pyramid_level(shape, kp, l)[b:b + 1, h:h + 1].double().cpu().numpy()
                                      for l in range(1, w.levels)]
        vl = [vh.double().numpy()] + [P.pyramid_level(shape, vp, l)[b:b + 1, h:h + 1].double().cpu().numpy()
                                      for l in range(1, w.levels)]
        o, l = O.attention(qh, kl, vl, mask[b:b + 1, h:h + 1].cpu(), w.block, w.sm_scale, w.causal, rows=row)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 2e-2 and mean <= 2e-3, (mode, policy, h, I, mx, mean)
    assert P.psa_get_device_status(ws) == P.PSA_OK
    check_band("wan14b full size, %s/%s" % (mode, policy), n_amb, n_pairs)


@pytest.mark.parametrize("name", ["wan14b", "qwen2.5vl", "wan1.3b"])
def test_fullsize_fp8_sampled(name):
    """The FP8 path (e4m3 Q and K) at the preset's full shape on its
    generated mask, checked on sampled query-block rows against the
    oracle's attention on the same e4m3 operands (the GPU's quantizer codes
    are pinned bit for bit in test_gpu_fp8.py; here the oracle quantizes
    the whole KV head itself), at the bf16 tolerances."""
    w = W.PRESETS[name]
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    kp, vp, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    mask, _ = run_mask(shape, params_for(w), q, k, bc)
    out = torch.empty_like(q)
    ws = P.workspace(P.psa_attention_fp8_workspace_bytes(shape), DEV)
    P.psa_attention_fwd_fp8(shape, q, k, v, kp, vp, mask, w.sm_scale, out, None, ws)
    torch.cuda.synchronize()
    assert P.psa_get_device_status(ws) == P.PSA_OK
    grp = w.Hq // w.Hkv
    rows = sample_rows(w, 10, seed=5)
    for (b, h), Is in by_head(rows).items():
        hrows = [(0, 0, I) for I in Is]
        kl = head_levels(shape, k, kp, b, h // grp, w.levels)
        vl = head_levels(shape, v, vp, b, h // grp, w.levels)
        o, _ = O.attention_fp8(q[b:b + 1, h:h + 1].cpu(), [x.astype(np.float32) for x in kl], vl,
                               mask[b:b + 1, h:h + 1].cpu(), w.block, w.sm_scale, w.causal, rows=hrows)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 2e-2 and mean <= 2e-3, (h, Is, mx, mean)


@pytest.mark.parametrize("name", ["wan14b", "qwen2.5vl", "wan1.3b"])
def test_fullsize_fp8_pv_sampled(name):
    """The FP8 path with e4m3 probabilities and values (reading R14) at the
    preset's full shape on its generated mask (Qwen2.5-VL: causal, 7 query
    heads per KV head, antidiagonal scorer with the cosine gate; Wan2.1-1.3B:
    64-token blocks, two query blocks per tile), on sampled
    query-block rows, against the oracle's attention_fp8(pv=True) on the
    whole KV head's levels (the value scale is per KV head), with the
    reference-shift tolerance of test_gpu_fp8.py (max-abs 5e-2, mean-abs
    5e-3)."""
    w = W.PRESETS[name]
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    kp, vp, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    mask, _ = run_mask(shape, params_for(w), q, k, bc)
    out = torch.empty_like(q)
    ws = P.workspace(P.psa_attention_fp8_workspace_bytes(shape), DEV)
    P.psa_attention_fwd_fp8_pv(shape, q, k, v, kp, vp, mask, w.sm_scale, out, None, ws)
    torch.cuda.synchronize()
    assert P.psa_get_device_status(ws) == P.PSA_OK
    rows = sample_rows(w, 10, seed=6)
    grp = w.Hq // w.Hkv
    worst = (0.0, 0.0)
    for (b, h), Is in by_head(rows).items():
        hrows = [(0, 0, I) for I in Is]
        kl = head_levels(shape, k, kp, b, h // grp, w.levels)
        vl = head_levels(shape, v, vp, b, h // grp, w.levels)
        o, _ = O.attention_fp8(q[b:b + 1, h:h + 1].cpu(), [x.astype(np.float32) for x in kl],
                               [x.astype(np.float32) for x in vl], mask[b:b + 1, h:h + 1].cpu(), w.block, w.sm_scale,
                               w.causal, rows=hrows, pv=True)
        mx, mean, _ = attn_errors(out[b:b + 1, h:h + 1], o)
        assert mx <= 5e-2 and mean <= 5e-3, (h, Is, mx, mean)
        worst = (max(worst[0], mx), max(worst[1], mean))
    note("fp8 P.V %s full size, sampled rows: vs the e4m3 oracle max %.2e mean %.2e" % ((name,) + worst))


def test_fullsize_backward_dq_wan14b_sampled():
    """The backward at the Wan2.1-14B shape at full grid: dq of sampled
    query blocks against the oracle's backward restricted to those blocks
    (a row's dq depends only on its own key set), same tolerance as the
    backward tests (max-abs 2e-2 of max|ref|, mean-abs 6e-3 of mean|ref|)."""
    w = W.PRESETS["wan14b"]
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    mask, _ = run_mask(shape, params_for(w), q, k)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    g = torch.Generator(device=DEV)
    g.manual_seed(11)
    dout = torch.randn(q.shape, generator=g, device=DEV).bfloat16()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = P.workspace(P.psa_attention_bwd_workspace_bytes(shape), DEV)
    P.psa_attention_bwd(shape, q, k, v, kp, vp, mask, w.sm_scale, out, lse, dout, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert P.psa_get_device_status(ws) == P.PSA_OK
    assert torch.isfinite(dk.float()).all() and torch.isfinite(dv.float()).all()
    rows = sample_rows(w, 6, seed=17)
    for (b, h), Is in by_head(rows).items():
        hrows = [(0, 0, I) for I in Is]
        rq, _, _ = O.attention_backward(q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, h:h + 1].cpu(),
                                        v[b:b + 1, h:h + 1].cpu(), mask[b:b + 1, h:h + 1].cpu(), w.block,
                                        w.sm_scale, False, w.levels, dout[b:b + 1, h:h + 1].cpu(), rows=hrows)
        for I in Is:
            sl = slice(I * w.block, min((I + 1) * w.block, w.N))
            ref = rq[0, 0, sl]
            got = dq[b, h, sl].double().cpu().numpy()
            err = np.abs(got - ref)
            assert err.max() <= 2e-2 * np.abs(ref).max() and err.mean() <= 6e-3 * np.abs(ref).mean(), \
                (h, I, err.max(), np.abs(ref).max(), err.mean(), np.abs(ref).mean())
