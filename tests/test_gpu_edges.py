"""GPU edge cases of the PSA path (through the C ABI), each against the oracle.

  * More than 1024 KV blocks: the mask generator's CTA-wide select kernel
    (the one-warp-per-row bucketed select takes at most 1024 keys per
    row), with both level
    policies and causal masking, and attention on the resulting mask.
  * Determinism of the mask (select kernel atomics) and of the FP8
    probability-and-value attention: repeated calls are bit-equal.
  * A bounded device wait that runs out: with the debug trap armed, every
    CTA of the attention kernel waits once on a barrier nothing arrives at
    (limit 1 ms), gives up, unwinds, and PSA_ERR_TIMEOUT with that wait's
    site comes back through psa_get_device_status; a normal call on the
    same workspace afterwards is correct.
"""
import re

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import video_transformers_b200 as P
import workloads as W
from amb_report import check_band
from psa_run import SKIP, attn_errors, levels_of, run_attention, run_mask, run_pyramid, shape_for

pytestmark = pytest.mark.gpu
DEV = "cuda"

TRAP_SITE = 10          # the attention kernel's debug trap wait


@pytest.mark.parametrize("policy,causal", [("mass", False), ("quantile", True)])
def test_select_over_1024_key_blocks(policy, causal):
    """N = 70,000 tokens in blocks of 64: 1094 KV blocks (the last holds 48
    tokens), beyond the one-warp-per-row select kernel's 1024."""
    N, d, block = 70000, 64, 64
    th = (0.6, 0.8, 0.9, 0.95) if policy == "mass" else (0.25, 0.5, 0.75, 0.875)
    w = W.Workload("nkb1094", B=1, Hq=2, Hkv=1, d=d, block=block, levels=4, causal=causal, dtype="bf16",
                   recipe="iid", n_iid=N, mask_mode="sample", thresholds=th, policy=policy, seed=81)
    q, k, v, _ = W.make_qkv(w, device="cpu")
    q = (q.float() * 2.0).bfloat16()                 # sharper softmax: masks with several levels
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    assert w.nqb == 1094
    shape = shape_for(w)
    pol = P.PSA_POLICY_QUANTILE if policy == "quantile" else P.PSA_POLICY_MASS
    params = P.make_params(P.PSA_MASK_SAMPLE, th, w.sm_scale, policy=pol)
    mask, mass = run_mask(shape, params, q, k)
    kp, vp, _ = run_pyramid(shape, k, v)
    out, lse, ws = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    Is = sorted({0, 1, 547, w.nqb - 2, w.nqb - 1, *rng.integers(0, w.nqb, size=11).tolist()})
    kl = levels_of(shape, kp, k)
    vl = levels_of(shape, vp, v)
    thf = [float(np.float32(t)) for t in th]
    n_amb = n_pairs = 0
    for h in range(w.Hq):
        rows = [(0, h, I) for I in Is]
        om = O.sampling_mass(q.cpu(), k.cpu(), block, w.sm_scale, causal, rows=rows)
        omask = O.make_mask(om, thf, 4, block, causal, rows=rows, policy=policy)
        if policy == "quantile":
            amb = O.ambiguous_pairs_quantile(om, thf, 4, causal, 1e-6, rows=rows)
        else:
            amb = O.ambiguous_pairs(om, thf, 1e-6, rows=rows)
        gm = mask.cpu().numpy()
        gmass = mass.cpu().numpy().astype(np.float64)
        for I in Is:
            o_row, g_row, a_row = om[0, h, I], gmass[0, h, I], amb[0, h, I]
            big = o_row > 1e-6
            assert (np.abs(g_row[big] - o_row[big]) / o_row[big]).max() <= 1e-4
            assert np.all((gm[0, h, I] == omask[0, h, I]) | a_row), (h, I)
            n_amb += int(a_row.sum())
            n_pairs += a_row.size
        levels_used = set(np.unique(gm[0, h, Is]).tolist())
        assert len(levels_used - {SKIP}) >= 2, levels_used
        o, l = O.attention(q.cpu(), kl, vl, mask.cpu(), block, w.sm_scale, causal, rows=rows)
        mx, mean, _ = attn_errors(out, o)
        assert mx <= 2e-2 and mean <= 2e-3, (h, mx, mean)
    check_band("nKB = 1094 select, %s" % policy, n_amb, n_pairs)
    assert P.psa_get_device_status(ws) == P.PSA_OK


def _tiny_attention_problem(seed=3):
    g = torch.Generator().manual_seed(seed)
    B, H, N, d, block = 1, 8, 2048, 128, 128
    q = torch.randn(B, H, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(B, H, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(B, H, N, d, generator=g).bfloat16().to(DEV)
    nb = N // block
    m = torch.randint(0, 4, (B, H, nb, nb), generator=g).to(torch.uint8).to(DEV)
    shape = P.make_shape(B, H, H, N, d, block, 4)
    return shape, q, k, v, m


def test_attention_wait_timeout_is_reported_and_recoverable():
    shape, q, k, v, mask = _tiny_attention_problem()
    kp, vp, _ = run_pyramid(shape, k, v)
    ws = P.workspace(P.psa_attention_workspace_bytes(shape), DEV)
    out = torch.empty_like(q)
    P.psa_debug_wait_control(ws, 1000000, trap=True)
    P.psa_attention_fwd(shape, q, k, v, kp, vp, mask, shape.d ** -0.5, out, None, ws)
    st = P.psa_get_device_status(ws)
    msg = P.psa_last_error()
    assert st == P.PSA_ERR_TIMEOUT, (st, msg)
    m = re.search(r"site (\d+), block (\d+), thread (\d+)", msg)
    assert m, msg
    site, blk, thr = (int(x) for x in m.groups())
    assert site == TRAP_SITE, msg
    assert 0 <= blk < 2 * torch.cuda.get_device_properties(0).multi_processor_count
    assert 0 <= thr < 192
    # the record was read and cleared; the debug words stay until reset
    assert P.psa_get_device_status(ws) == P.PSA_OK
    P.psa_debug_wait_control(ws, 0, trap=False)
    out2, lse2, _ = run_attention(shape, q, k, v, kp, vp, mask, shape.d ** -0.5, ws=ws)
    torch.cuda.synchronize()
    ws2 = P.workspace(P.psa_attention_workspace_bytes(shape), DEV)
    ref, ref_lse, _ = run_attention(shape, q, k, v, kp, vp, mask, shape.d ** -0.5, ws=ws2)
    assert torch.equal(out2, ref) and torch.equal(lse2, ref_lse)
    kl, vl = levels_of(shape, kp, k), levels_of(shape, vp, v)
    rows = [(0, h, I) for h in (0, 5) for I in range(shape.N // shape.block)]
    o, _ = O.attention(q, kl, vl, mask.cpu(), shape.block, shape.d ** -0.5, False, rows=rows)
    mx, mean, _ = attn_errors(out2, o)
    assert mx <= 2e-2 and mean <= 2e-3, (mx, mean)


@pytest.mark.parametrize("name,heads,policy", [("wan14b", (1, 1), P.PSA_POLICY_MASS),
                                               ("wan1.3b", (2, 2), P.PSA_POLICY_QUANTILE),
                                               ("qwen2.5vl", (7, 1), P.PSA_POLICY_MASS)])
def test_mask_is_deterministic(name, heads, policy):
    """Three calls of psa_make_mask give the same mask and masses bit for
    bit, at the presets' full sequence lengths (591, 512 and 256 key
    blocks): the select kernel's shared-memory atomics add integers (counts
    and fixed-point sums, the same in any order) or place a block in its
    bucket's list, whose order the exact count does not depend on."""
    from psa_run import params_for
    w = W.PRESETS[name].replace(Hq=heads[0], Hkv=heads[1])
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    _, _, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    runs = [run_mask(shape, params_for(w, policy), q, k, bc) for _ in range(3)]
    for m, s in runs[1:]:
        assert torch.equal(m, runs[0][0]) and torch.equal(s, runs[0][1])


def test_fp8_pv_attention_is_deterministic():
    """Two calls of the FP8 probability-and-value path give the same output
    and lse bit for bit (no atomics; a fixed order of work per query tile)."""
    w = W.reduced("wan14b", grid=(4, 12, 16), heads=(2, 2))
    q, k, v, _ = W.make_qkv(w, device=DEV)
    shape = shape_for(w)
    kp, vp, _ = run_pyramid(shape, k, v)
    from psa_run import params_for
    mask, _ = run_mask(shape, params_for(w), q, k)
    outs = []
    for _ in range(2):
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
        ws = P.workspace(P.psa_attention_fp8_workspace_bytes(shape), DEV)
        P.psa_attention_fwd_fp8_pv(shape, q, k, v, kp, vp, mask, w.sm_scale, out, lse, ws)
        torch.cuda.synchronize()
        assert P.psa_get_device_status(ws) == P.PSA_OK
        outs.append((out, lse))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
