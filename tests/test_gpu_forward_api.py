"""psa_forward (the whole path in one call) against the stage-by-stage
calls it sequences: the same kernels on the same inputs, so the mask and the
output must be bit-equal."""
import pytest
import torch

import video_transformers_b200 as P
import workloads as W
from psa_run import MODES, params_for, run_attention, run_mask, run_pyramid, shape_for

pytestmark = pytest.mark.gpu
DEV = "cuda"


def stage_by_stage(w, q, k, v, precision):
    shape = shape_for(w)
    kp, vp, bc = run_pyramid(shape, k, v, with_cos=w.cos_min > -2)
    mask, _ = run_mask(shape, params_for(w), q, k, bc)
    if precision == "bf16":
        out, lse, _ = run_attention(shape, q, k, v, kp, vp, mask, w.sm_scale)
    else:
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
        ws = P.workspace(P.psa_attention_fp8_workspace_bytes(shape), DEV)
        P.psa_attention_fwd_fp8_pv(shape, q, k, v, kp, vp, mask, w.sm_scale, out, lse, ws)
        torch.cuda.synchronize()
    return out, mask, lse


@pytest.mark.parametrize("name,precision", [("wan14b", "bf16"), ("qwen2.5vl", "bf16"), ("wan14b", "fp8_pv"),
                                            ("wan1.3b", "bf16")])
def test_psa_forward_equals_the_stage_calls(name, precision):
    w = W.reduced(name, grid=(4, 12, 16), heads=(4, 4) if name != "qwen2.5vl" else (7, 1))
    q, k, v, _ = W.make_qkv(w, device=DEV)
    ref_out, ref_mask, ref_lse = stage_by_stage(w, q, k, v, precision)
    out, mask, lse = P.psa_forward(q, k, v, block=w.block, levels=w.levels, thresholds=w.thresholds,
                                   mode=MODES[w.mask_mode], causal=w.causal, sm_scale=w.sm_scale, stride=w.stride,
                                   cos_min=w.cos_min, n_dense_prefix=w.n_dense_prefix, precision=precision,
                                   want_lse=True)
    torch.cuda.synchronize()
    assert P.psa_forward_status() == P.PSA_OK
    assert torch.equal(mask, ref_mask)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_psa_forward_with_a_given_mask():
    w = W.reduced("wan14b", grid=(4, 12, 16), heads=(2, 2))
    q, k, v, _ = W.make_qkv(w, device=DEV)
    ref_out, ref_mask, _ = stage_by_stage(w, q, k, v, "bf16")
    out, mask, _ = P.psa_forward(q, k, v, block=w.block, levels=w.levels, thresholds=w.thresholds,
                                 sm_scale=w.sm_scale, mask=ref_mask)
    torch.cuda.synchronize()
    assert mask is ref_mask and torch.equal(out, ref_out)
