"""Parity of the backward pass (psa_attention_bwd, through the C ABI) with the
oracle's attention_backward, which is pinned by torch autograd, finite
differences and the dense special case (tests/test_oracle_pins.py).

Tolerance, per gradient (dq, dk, dv) against the fp64 oracle on the same
bf16 inputs: max-abs error <= 2e-2 * max|ref| and mean-abs error <= 6e-3 *
mean|ref|.  The GPU rounds P and dZ to bf16 (relative 2^-9) before their
products, reads the bf16 pyramid levels (the oracle pools in fp64) and the
bf16 forward output in D = dO.O, and rounds the result to bf16 (alone a
mean error of about 0.15 % of mean|ref| on these inputs).  Measured on
B200 over the cases below: at most 1.07 % of max|ref| and 0.30 % of
mean|ref|, so the bounds leave a margin of about 2x.  Rows and tokens that nothing
reaches must come back as exact zeros."""
import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import video_transformers_b200 as P
import workloads as W
from amb_report import note
from psa_run import SKIP, params_for, run_attention, run_mask, run_pyramid, shape_for

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_MAX, REL_MEAN = 2e-2, 6e-3


def gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def run_backward(shape, q, k, v, kp, vp, mask, sm_scale, out, lse, dout):
    dq, dk, dv = torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
    ws = P.workspace(P.psa_attention_bwd_workspace_bytes(shape), q.device)
    L1 = shape.levels > 1
    P.psa_attention_bwd(shape, q, k, v, kp if L1 else None, vp if L1 else None, mask.contiguous(), sm_scale, out, lse,
                        dout, dq, dk, dv, ws)
    st = P.psa_get_device_status(ws)
    assert st == P.PSA_OK, P.psa_last_error()
    torch.cuda.synchronize()
    return dq, dk, dv


def compare(name, got, ref):
    g = got.double().cpu().numpy()
    assert np.isfinite(g).all(), name
    err = np.abs(g - ref)
    mx, mean = err.max(), err.mean()
    scale_mx, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    note("backward %s: max-abs %.3g (%.4f of max|ref| %.3g), mean-abs %.3g (%.4f of mean|ref| %.3g)"
         % (name, mx, mx / scale_mx, scale_mx, mean, mean / scale_mean, scale_mean))
    assert mx <= REL_MAX * scale_mx and mean <= REL_MEAN * scale_mean, \
        (name, mx, mean, scale_mx, scale_mean, mx / scale_mx, mean / scale_mean)
    return mx / scale_mx, mean / scale_mean


def full_check(shape, q, k, v, mask, causal, seed=0):
    sm_scale = shape.d ** -0.5
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, sm_scale)
    g = gen(seed + 1000)
    dout = torch.randn(q.shape, generator=g).bfloat16().to(DEV)
    dq, dk, dv = run_backward(shape, q, k, v, kp, vp, mask, sm_scale, out, lse, dout)
    rq, rk, rv = O.attention_backward(q, k, v, mask.cpu(), shape.block, sm_scale, causal, shape.levels, dout)
    res = {n: compare(n, a, b) for n, a, b in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv))}
    return dq, dk, dv, res


@pytest.mark.parametrize("block,d,causal,L,N,heads", [
    (128, 128, False, 4, 1000, (2, 1)),      # GQA 2:1, ragged last block (104 tokens)
    (128, 64, True, 4, 520, (4, 2)),         # causal, ragged
    (64, 128, True, 4, 456, (2, 2)),         # 64-token blocks: two query blocks per tile
    (64, 64, False, 3, 300, (3, 1)),         # GQA 3:1, L = 3
    (128, 128, False, 1, 256, (1, 1)),       # binary mask, level 0 only
    (64, 128, False, 2, 70, (2, 2)),         # shorter than one query tile
    (128, 128, True, 2, 72, (1, 1)),
])
def test_backward_random_masks(block, d, causal, L, N, heads):
    g = gen(21)
    Hq, Hkv = heads
    B = 2
    q = torch.randn(B, Hq, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(B, Hkv, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(B, Hkv, N, d, generator=g).bfloat16().to(DEV)
    nb = -(-N // block)
    m = torch.randint(0, L + 1, (B, Hq, nb, nb), generator=g)
    mask = torch.where(m == L, torch.full_like(m, SKIP), m).to(torch.uint8)
    mask[0, 0, 0] = SKIP                       # an all-skip query block: dq rows exactly 0
    shape = P.make_shape(B, Hq, Hkv, N, d, block, L, causal)
    dq, dk, dv, _ = full_check(shape, q, k, v, mask.to(DEV), causal)
    assert torch.all(dq[0, 0, :min(block, N)] == 0)


def test_backward_level0_is_dense_autograd():
    """All level 0: the gradients of plain softmax attention, from torch
    autograd through SDPA in float64."""
    g = gen(31)
    N, d, block = 640, 128, 128
    q = torch.randn(1, 2, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(1, 2, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(1, 2, N, d, generator=g).bfloat16().to(DEV)
    nb = N // block
    mask = torch.zeros(1, 2, nb, nb, dtype=torch.uint8, device=DEV)
    shape = P.make_shape(1, 2, 2, N, d, block, 4)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, d ** -0.5)
    dout = torch.randn(q.shape, generator=g).bfloat16().to(DEV)
    dq, dk, dv = run_backward(shape, q, k, v, kp, vp, mask, d ** -0.5, out, lse, dout)
    qt, kt, vt = (x.double().cpu().requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=d ** -0.5)
    o.backward(dout.double().cpu())
    for n, a, b in (("dq", dq, qt.grad), ("dk", dk, kt.grad), ("dv", dv, vt.grad)):
        compare(n, a, b.numpy())


def test_backward_unused_kv_tokens_get_zero():
    """A KV block no query uses at any level gets exactly zero gradient."""
    g = gen(41)
    N, d, block = 1024, 128, 128
    q = torch.randn(1, 2, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(1, 2, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(1, 2, N, d, generator=g).bfloat16().to(DEV)
    nb = N // block
    mask = torch.randint(0, 4, (1, 2, nb, nb), generator=g).to(torch.uint8)
    J = 5
    mask[:, :, :, J] = SKIP
    shape = P.make_shape(1, 2, 2, N, d, block, 4)
    dq, dk, dv, _ = full_check(shape, q, k, v, mask.to(DEV), False)
    sl = slice(J * block, (J + 1) * block)
    assert torch.all(dk[:, :, sl] == 0) and torch.all(dv[:, :, sl] == 0)


@pytest.mark.parametrize("name,grid,heads", [("wan14b", (3, 9, 16), (2, 2)), ("qwen2.5vl", (6, 8, 16), (7, 1)),
                                             ("wan1.3b", (3, 10, 12), (2, 2))])
def test_backward_on_generated_masks(name, grid, heads):
    """The whole forward path (pyramid, generated mask, attention), then the
    backward on its mask."""
    w = W.reduced(name, grid=grid, heads=heads)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    shape = shape_for(w)
    _, _, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    mask, _ = run_mask(shape, params_for(w), q, k, bc)
    full_check(shape, q, k, v, mask, w.causal, seed=3)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64)])
def test_backward_many_items_per_cta(d, block):
    """More query tiles and KV tiles than SMs: every CTA of both persistent
    kernels takes several items; checked on a subset of heads."""
    g = gen(71)
    H, N = 40, 1024
    q = torch.randn(1, H, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(1, H, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(1, H, N, d, generator=g).bfloat16().to(DEV)
    nb = N // block
    m = torch.randint(0, 5, (1, H, nb, nb), generator=g)
    mask = torch.where(m == 4, torch.full_like(m, SKIP), m).to(torch.uint8).to(DEV)
    shape = P.make_shape(1, H, H, N, d, block, 4)
    sm_scale = d ** -0.5
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, sm_scale)
    dout = torch.randn(q.shape, generator=g).bfloat16().to(DEV)
    dq, dk, dv = run_backward(shape, q, k, v, kp, vp, mask, sm_scale, out, lse, dout)
    hs = [0, 13, 39]
    sel = lambda x: x[:, hs].contiguous()
    rq, rk, rv = O.attention_backward(sel(q), sel(k), sel(v), sel(mask).cpu(), block, sm_scale, False, 4, sel(dout))
    for n, a, b in (("dq", sel(dq), rq), ("dk", sel(dk), rk), ("dv", sel(dv), rv)):
        compare(n, a, b)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64)])
def test_backward_is_deterministic(d, block):
    """Three calls on the same inputs give bit-identical gradients (the
    kernels have no atomics and a fixed order of work inside every tile;
    a race between the warps that share a TMEM buffer would show here)."""
    g = gen(81)
    H, N = 40, 1024
    q = torch.randn(1, H, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(1, H, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(1, H, N, d, generator=g).bfloat16().to(DEV)
    nb = N // block
    m = torch.randint(0, 5, (1, H, nb, nb), generator=g)
    mask = torch.where(m == 4, torch.full_like(m, SKIP), m).to(torch.uint8).to(DEV)
    shape = P.make_shape(1, H, H, N, d, block, 4)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, d ** -0.5)
    dout = torch.randn(q.shape, generator=g).bfloat16().to(DEV)
    first = run_backward(shape, q, k, v, kp, vp, mask, d ** -0.5, out, lse, dout)
    for _ in range(2):
        again = run_backward(shape, q, k, v, kp, vp, mask, d ** -0.5, out, lse, dout)
        for a, b in zip(first, again):
            assert torch.equal(a, b)
