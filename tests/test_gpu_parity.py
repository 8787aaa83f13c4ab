"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Tolerances: pyramid fp32 max-abs 1e-6, bf16 within 1 bf16 ulp of the fp64
mean; block cosine 1e-5; block mass relative 1e-4 (where the mass is above
1e-6); masks bit-exact except pairs the oracle marks ambiguous (a threshold
within 1e-6 of the range near-equal masses allow); attention output max-abs
2e-2 and mean-abs 2e-3 against the oracle in fp64, lse abs 2e-2.
Each stage is fed the same inputs on both sides: the GPU pyramid and mask
are passed to the oracle's later stages as well as recomputed there."""
import math

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import video_transformers_b200 as P
import workloads as W
from amb_report import check_band
from psa_run import (SKIP, attn_errors, bf16_ulp, levels_of, params_for, run_attention, run_mask,
                     run_pyramid, shape_for)

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def randn(g, *shape, dtype=torch.bfloat16):
    return torch.randn(*shape, generator=g).to(dtype).to(DEV)


# --------------------------------------------------------------------------------------
# stage 1
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("L,d,N", [(4, 64, 1024), (4, 128, 200), (3, 128, 332), (2, 64, 90)])
def test_pyramid_parity(dtype, L, d, N):
    g = gen(11)
    k, v = randn(g, 2, 3, N, d, dtype=dtype), randn(g, 2, 3, N, d, dtype=dtype)
    s = P.make_shape(2, 3, 3, N, d, 64, L, dtype=P.PSA_DT_FP32 if dtype == torch.float32 else P.PSA_DT_BF16)
    kp, vp, _ = run_pyramid(s, k, v)
    torch.cuda.synchronize()
    ok_bits = total = 0
    for t, buf in ((k, kp), (v, vp)):
        got = levels_of(s, buf, t)
        for l in range(1, L):
            want = O.pool_level(t, l)
            if dtype == torch.float32:
                assert np.abs(got[l] - want).max() <= 1e-6
            else:
                err = np.abs(got[l] - want)
                assert np.all(err <= bf16_ulp(want) + 1e-30)
                rne = torch.tensor(want).to(torch.bfloat16).double().numpy()
                ok_bits += int((got[l] == rne).sum())
                total += rne.size
    if dtype == torch.bfloat16:
        assert ok_bits / total > 0.99          # single rounding of an (almost always) exact fp32 sum


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("block,N,d", [(64, 200, 64), (128, 300, 128), (128, 129, 64)])
def test_blockcos_parity(dtype, block, N, d):
    g = gen(12)
    k = randn(g, 1, 2, N, d, dtype=dtype)
    k[0, 1, 3] = 0.0                                           # zero key
    k[0, 0, 64:80] = k[0, 0, 64:65] * 2.0                      # near-parallel run
    s = P.make_shape(1, 2, 2, N, d, block, 1, dtype=P.PSA_DT_FP32 if dtype == torch.float32 else P.PSA_DT_BF16)
    _, _, bc = run_pyramid(s, k, k, with_cos=True)
    want = O.block_cosine(k, block)
    assert np.abs(bc.cpu().numpy() - want).max() <= 1e-5


# --------------------------------------------------------------------------------------
# stage 2
# --------------------------------------------------------------------------------------

def check_mask(w, q, k, rows=None):
    shape, params = shape_for(w), params_for(w)
    bc = None
    if w.cos_min > -2:
        _, _, bc = run_pyramid(shape, k, k, with_cos=True) if shape.levels == 1 else \
            (None, None, run_pyramid(shape, k, k.clone(), with_cos=True)[2])
    mask, mass = run_mask(shape, params, q, k, bc)
    mask, mass = mask.cpu().numpy(), mass.cpu().numpy().astype(np.float64)
    if w.mask_mode == "sample":
        om = O.sampling_mass(q, k, w.block, w.sm_scale, w.causal, rows=rows)
    else:
        om = O.antidiag_mass(q, k, w.block, w.stride, w.sm_scale, w.causal, rows=rows)
    cos = None if bc is None else bc.cpu().numpy().astype(np.float64)
    omask = O.make_mask(om, w.thresholds, w.levels, w.block, w.causal, w.n_dense_prefix, cos, w.cos_min,
                        w.Hq // w.Hkv, rows=rows)
    amb = O.ambiguous_pairs(om, w.thresholds, 1e-6, rows, cos, w.cos_min, w.Hq // w.Hkv)
    sel = ~np.isnan(om)
    big = sel & (om > 1e-6)
    rel = np.abs(mass[big] - om[big]) / om[big]
    assert rel.max() <= 1e-4, rel.max()
    bad = sel & ~amb & (mask != omask)
    assert bad.sum() == 0, "mask mismatches outside the ambiguity band: %d (ambiguous %d)" % (bad.sum(), (amb & sel).sum())
    check_band("%s %s N=%d" % (w.name, w.mask_mode, w.N), int((amb & sel).sum()), int(sel.sum()))
    return mask, int((amb & sel).sum()), int(sel.sum())


@pytest.mark.parametrize("name,grid,heads,n_text", [
    ("wan1.3b", (3, 10, 12), (2, 2), None),          # N = 360: ragged last block of 40
    ("cogvideox5b", (3, 10, 15), (3, 3), 30),         # text prefix, N = 480: ragged last block of 32
    ("wan14b", (4, 12, 16), (2, 2), None),           # block 128, N = 768
    ("wan14b", (3, 9, 16), (2, 2), None),            # N = 432: ragged
])
def test_mask_sampling_parity(name, grid, heads, n_text):
    w = W.reduced(name, grid=grid, heads=heads, n_text=n_text)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    check_mask(w, q.to(DEV), k.to(DEV))


def test_mask_sampling_causal_gqa():
    w = W.reduced("wan14b", grid=(3, 8, 16), heads=(4, 2)).replace(causal=True)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    mask, _, _ = check_mask(w, q.to(DEV), k.to(DEV))
    nb = mask.shape[-1]
    assert np.all(mask[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] == SKIP)


@pytest.mark.parametrize("cos_min", [0.8, -3.0, 0.1])
def test_mask_antidiag_parity(cos_min):
    w = W.reduced("qwen2.5vl", grid=(6, 8, 16), heads=(7, 1)).replace(cos_min=cos_min)   # N = 768
    q, k, v, _ = W.make_qkv(w, device="cpu")
    check_mask(w, q.to(DEV), k.to(DEV))


def test_mask_antidiag_noncausal_block64():
    w = W.reduced("qwen2.5vl", grid=(5, 8, 10), heads=(2, 2)).replace(causal=False, block=64, cos_min=-3.0)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    check_mask(w, q.to(DEV), k.to(DEV))


# --------------------------------------------------------------------------------------
# stage 3
# --------------------------------------------------------------------------------------

def oracle_attention_from_gpu(w, q, k, v, kp, vp, mask, rows=None):
    shape = shape_for(w)
    kl = levels_of(shape, kp, k) if w.levels > 1 else [k.double().cpu().numpy()]
    vl = levels_of(shape, vp, v) if w.levels > 1 else [v.double().cpu().numpy()]
    return O.attention(q, kl, vl, mask.cpu(), w.block, w.sm_scale, w.causal, rows=rows)


def full_path(w, q, k, v, mask=None):
    shape = shape_for(w)
    kp, vp, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    if mask is None:
        mask, _ = run_mask(shape, params_for(w), q, k, bc)
    out, lse, ws = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    return kp, vp, mask, out, lse, ws


def assert_attn(w, q, k, v, kp, vp, mask, out, lse, rows=None):
    o, l = oracle_attention_from_gpu(w, q, k, v, kp, vp, mask, rows)
    mx, mean, n = attn_errors(out, o)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    lg = lse.cpu().numpy().astype(np.float64)
    sel = ~np.isnan(l)
    fin = sel & np.isfinite(l)
    assert np.all(np.isneginf(lg[sel & ~np.isfinite(l)]))
    assert np.abs(lg[fin] - l[fin]).max() <= 2e-2
    return mx, mean


def test_attention_tiny_given_mask():
    """The tiny fp32 case: B1 H2 N1024 d64, a drawn mask over {0,1,2,3,SKIP}."""
    w = W.PRESETS["tiny"]
    q, k, v, g = W.make_qkv(w, device="cpu")
    mask = W.make_given_mask(w, g)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask.to(DEV), w.sm_scale)
    # oracle from the exact fp32 inputs, its own pyramid
    kl, vl = O.build_pyramid(k, v, w.levels)
    o, l = O.attention(q, kl, vl, mask, w.block, w.sm_scale, w.causal)
    mx, mean, _ = attn_errors(out, o)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("name,grid,heads,n_text", [
    ("wan1.3b", (3, 10, 12), (2, 2), None),
    ("cogvideox5b", (3, 10, 15), (2, 2), 30),
    ("qwen2.5vl", (6, 8, 16), (7, 1), None),
    ("wan14b", (4, 12, 16), (2, 2), None),
    ("wan14b", (3, 9, 16), (2, 2), None),
])
def test_attention_pipeline_parity(name, grid, heads, n_text):
    w = W.reduced(name, grid=grid, heads=heads, n_text=n_text)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    kp, vp, mask, out, lse, _ = full_path(w, q, k, v)
    assert_attn(w, q, k, v, kp, vp, mask, out, lse)


@pytest.mark.parametrize("block,d,causal,L,N,heads", [
    (128, 128, False, 4, 1000, (2, 1)),
    (128, 64, True, 4, 520, (4, 2)),
    (64, 128, True, 4, 456, (2, 2)),
    (64, 64, False, 3, 300, (3, 1)),
    (128, 128, False, 1, 256, (1, 1)),
    (64, 128, False, 2, 70, (2, 2)),
    (128, 128, True, 2, 72, (1, 1)),
])
def test_attention_random_masks(block, d, causal, L, N, heads):
    g = gen(21)
    Hq, Hkv = heads
    w = W.Workload("rand", B=2, Hq=Hq, Hkv=Hkv, d=d, block=block, levels=L, causal=causal, dtype="bf16",
                   recipe="iid", n_iid=N)
    q, k, v = randn(g, 2, Hq, N, d), randn(g, 2, Hkv, N, d), randn(g, 2, Hkv, N, d)
    nb = -(-N // block)
    m = torch.randint(0, L + 1, (2, Hq, nb, nb), generator=g)
    mask = torch.where(m == L, torch.full_like(m, SKIP), m).to(torch.uint8)
    mask[0, 0, 0] = SKIP                       # an all-skip row
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask.to(DEV), w.sm_scale)
    assert_attn(w, q, k, v, kp, vp, mask, out, lse)
    assert torch.all(out[0, 0, :min(block, N)] == 0)


@pytest.mark.parametrize("block,d", [(128, 128), (64, 64)])
def test_attention_level0_is_dense(block, d):
    g = gen(31)
    N = 640
    q, k, v = randn(g, 1, 2, N, d), randn(g, 1, 2, N, d), randn(g, 1, 2, N, d)
    nb = -(-N // block)
    mask = torch.zeros(1, 2, nb, nb, dtype=torch.uint8, device=DEV)
    shape = P.make_shape(1, 2, 2, N, d, block, 4)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, d ** -0.5)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(), scale=d ** -0.5)
    err = (out.double() - ref).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


def test_attention_skip_ignores_nan():
    g = gen(41)
    N, d, block = 1024, 128, 128
    q, k, v = randn(g, 1, 2, N, d), randn(g, 1, 2, N, d), randn(g, 1, 2, N, d)
    nb = N // block
    m = torch.randint(0, 4, (1, 2, nb, nb), generator=g).to(torch.uint8)
    J = 5
    rows_skip = [0, 2, 3]
    for I in rows_skip:
        m[:, :, I, J] = SKIP
    mask = m.to(DEV)
    shape = P.make_shape(1, 2, 2, N, d, block, 4)
    kp, vp, _ = run_pyramid(shape, k, v)
    out1, lse1, _ = run_attention(shape, q, k, v, kp, vp, mask, d ** -0.5)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, J * block:(J + 1) * block] = float("nan")
    v2[:, :, J * block:(J + 1) * block] = float("nan")
    kp2, vp2, _ = run_pyramid(shape, k2, v2)
    out2, lse2, _ = run_attention(shape, q, k2, v2, kp2, vp2, mask, d ** -0.5)
    for I in rows_skip:
        sl = slice(I * block, (I + 1) * block)
        assert torch.equal(out1[:, :, sl], out2[:, :, sl])
        assert torch.equal(lse1[:, :, sl], lse2[:, :, sl])
    assert torch.isnan(out2[:, :, 1 * block:2 * block]).all()


def test_attention_identical_groups_any_level_is_dense():
    g = gen(51)
    N, d, block = 768, 128, 128
    base_k, base_v = randn(g, 1, 2, N // 8, d), randn(g, 1, 2, N // 8, d)
    k = base_k.repeat_interleave(8, dim=2).contiguous()
    v = base_v.repeat_interleave(8, dim=2).contiguous()
    q = randn(g, 1, 2, N, d)
    nb = N // block
    mask = torch.randint(0, 4, (1, 2, nb, nb), generator=g).to(torch.uint8).to(DEV)
    shape = P.make_shape(1, 2, 2, N, d, block, 4)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, _, _ = run_attention(shape, q, k, v, kp, vp, mask, d ** -0.5)
    out_again, _, _ = run_attention(shape, q, k, v, kp, vp, mask, d ** -0.5)
    assert torch.equal(out, out_again)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(), scale=d ** -0.5)
    err = (out.double() - ref).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


def test_attention_plan_stats_and_status():
    g = gen(61)
    N, d, block = 512, 64, 64
    q, k, v = randn(g, 1, 1, N, d), randn(g, 1, 1, N, d), randn(g, 1, 1, N, d)
    nb = N // block
    mask = torch.full((1, 1, nb, nb), SKIP, dtype=torch.uint8)
    mask[0, 0, :, 0] = 0       # 64 rows each
    mask[0, 0, :, 1] = 3       # 8 rows each
    shape = P.make_shape(1, 1, 1, N, d, block, 4)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, ws = run_attention(shape, q, k, v, kp, vp, mask.to(DEV), d ** -0.5)
    nt, nr = P.psa_attention_plan_stats(shape, ws)
    # 4 query tiles of two 64-row blocks: both halves agree -> one 64-row and one 8-row segment
    assert nr == 4 * (64 + 8) and nt == 4
    assert P.psa_get_device_status(ws) == P.PSA_OK


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64)])
def test_attention_many_items_per_cta_with_rescale(d, block):
    """More query tiles than SMs (every CTA of the persistent grid takes
    several items), and keys of the late KV blocks scaled up so the running
    max of some rows of a warp jumps by more than the lazy-rescale threshold
    while others do not."""
    g = gen(71)
    H, N = 40, 1024
    q, k, v = randn(g, 1, H, N, d), randn(g, 1, H, N, d), randn(g, 1, H, N, d)
    k[:, :, N // 2:] *= 6.0
    nb = N // block
    m = torch.randint(0, 5, (1, H, nb, nb), generator=g)
    mask = torch.where(m == 4, torch.full_like(m, SKIP), m).to(torch.uint8)
    mask[:, :, :, nb - 1] = 0
    w = W.Workload("many", B=1, Hq=H, Hkv=H, d=d, block=block, levels=4, causal=False, dtype="bf16",
                   recipe="iid", n_iid=N)
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask.to(DEV), w.sm_scale)
    rows = [(0, h, I) for h in range(0, H, 7) for I in range(nb)]
    assert_attn(w, q, k, v, kp, vp, mask, out, lse, rows=rows)
