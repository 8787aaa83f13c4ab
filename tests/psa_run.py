"""Test helpers: run the CUDA path through the Python binding of the C ABI,
and compare its results with the oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import video_transformers_b200 as P
import workloads as W

SKIP = 0xFF


def run_pyramid(w_or_shape, k, v, with_cos=False):
    shape = w_or_shape
    kp, vp = P.pyramid_buffers(shape, k.device, k.dtype)
    nkb = -(-shape.N // shape.block)
    bc = torch.empty(shape.B, shape.Hkv, nkb, dtype=torch.float32, device=k.device) if with_cos else None
    P.psa_build_pyramid(shape, k, v, kp if shape.levels > 1 else None, vp if shape.levels > 1 else None, bc)
    return kp, vp, bc


def levels_of(shape, buf, tensor0):
    """[level 0 (the input), level 1, ...] as float64 numpy arrays."""
    out = [tensor0.double().cpu().numpy()]
    for l in range(1, shape.levels):
        out.append(P.pyramid_level(shape, buf, l).double().cpu().numpy())
    return out


def run_mask(shape, params, q, k, blockcos=None):
    nb = -(-shape.N // shape.block)
    mask = torch.empty(shape.B, shape.Hq, nb, nb, dtype=torch.uint8, device=q.device)
    mass = torch.empty(shape.B, shape.Hq, nb, nb, dtype=torch.float32, device=q.device)
    ws = P.workspace(P.psa_mask_workspace_bytes(shape, params), q.device)
    P.psa_make_mask(shape, params, q, k, blockcos, mask, mass, ws)
    st = P.psa_get_device_status(ws)
    assert st == P.PSA_OK, "device status %d" % st
    return mask, mass


def run_attention(shape, q, k, v, kp, vp, mask, sm_scale, want_lse=True, ws=None):
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    if ws is None:
        ws = P.workspace(P.psa_attention_workspace_bytes(shape), q.device)
    L1 = shape.levels > 1
    P.psa_attention_fwd(shape, q, k, v, kp if L1 else None, vp if L1 else None, mask.contiguous(), sm_scale, out,
                        lse, ws)
    st = P.psa_get_device_status(ws)
    assert st == P.PSA_OK, "device status %d" % st
    return out, lse, ws


MODES = {"sample": P.PSA_MASK_SAMPLE, "antidiag": P.PSA_MASK_ANTIDIAG, "meankey": P.PSA_MASK_MEANKEY}


def params_for(w: W.Workload, policy: int = P.PSA_POLICY_MASS):
    return P.make_params(MODES[w.mask_mode], w.thresholds, w.sm_scale, stride=w.stride, cos_min=w.cos_min,
                         n_dense_prefix=w.n_dense_prefix, policy=policy)


def shape_for(w: W.Workload):
    return P.make_shape(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.levels, w.causal,
                        P.PSA_DT_FP32 if w.dtype == "fp32" else P.PSA_DT_BF16)


def attn_errors(gpu_out, ora_out, rows_mask=None):
    """max-abs and mean-abs of gpu - oracle over the rows the oracle computed."""
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    o = np.asarray(ora_out)
    sel = ~np.isnan(o[..., 0])
    if rows_mask is not None:
        sel &= rows_mask
    diff = np.abs(g[sel] - o[sel])
    return float(diff.max()), float(diff.mean()), int(sel.sum())


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 1e-38)
    e = np.floor(np.log2(ax))
    return 2.0 ** (e - 7)
