"""Python binding of libpsa.so, the B200 (sm_100a) PSA forward path.

Argument marshalling only: every function below has the name of the C entry
point it calls (include/psa.h), takes torch tensors that already live on the
GPU, passes their device pointers and the current CUDA stream, and raises
:class:`PsaError` on a non-zero status.  All computation happens in the CUDA
kernels of libpsa.so; there is no CPU fallback.  If the library has not been
built (``python -m video_transformers_b200.build``) the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsa.so")

PSA_OK, PSA_ERR_INVALID_ARG, PSA_ERR_UNSUPPORTED, PSA_ERR_WORKSPACE, PSA_ERR_CUDA, PSA_ERR_TIMEOUT = range(6)
PSA_DT_BF16, PSA_DT_FP32 = 0, 1
PSA_MASK_SAMPLE, PSA_MASK_ANTIDIAG, PSA_MASK_MEANKEY = 0, 1, 2
PSA_POLICY_MASS, PSA_POLICY_QUANTILE = 0, 1
PSA_SKIP = 0xFF

EXPORTS = [
    "psa_pyramid_bytes", "psa_pyramid_level_offset", "psa_build_pyramid",
    "psa_mask_workspace_bytes", "psa_make_mask",
    "psa_attention_workspace_bytes", "psa_attention_fwd", "psa_attention_fwd_static", "psa_attention_plan_stats",
    "psa_attention_bwd_workspace_bytes", "psa_attention_bwd",
    "psa_quantize_qk_fp8", "psa_attention_fp8_workspace_bytes", "psa_attention_fwd_fp8", "psa_attention_fwd_fp8_pv",
    "psa_get_device_status", "psa_get_static_device_status", "psa_debug_wait_control",
    "psa_last_error", "psa_version",
]


class PsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("psa status %d: %s" % (status, msg))
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("block", ctypes.c_int32),
                ("levels", ctypes.c_int32), ("causal", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class MaskParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("n_samples", ctypes.c_int32), ("stride", ctypes.c_int32),
                ("thresholds", ctypes.c_float * 8), ("n_thresholds", ctypes.c_int32),
                ("cos_min", ctypes.c_float), ("n_dense_prefix", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("policy", ctypes.c_int32)]


def _load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError("libpsa.so is not built (run: python -m video_transformers_b200.build); "
                          "the PSA path has no CPU fallback")
    lib = ctypes.CDLL(path)
    P, S, I, F, Z = ctypes.c_void_p, ctypes.POINTER(Shape), ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    MP = ctypes.POINTER(MaskParams)
    sig = {
        "psa_pyramid_bytes": (Z, [S]),
        "psa_pyramid_level_offset": (Z, [S, ctypes.c_int]),
        "psa_build_pyramid": (I, [S, P, P, P, P, P, P]),
        "psa_mask_workspace_bytes": (Z, [S, MP]),
        "psa_make_mask": (I, [S, MP, P, P, P, P, P, P, Z, P]),
        "psa_attention_workspace_bytes": (Z, [S]),
        "psa_attention_fwd": (I, [S, P, P, P, P, P, P, F, P, P, P, Z, P]),
        "psa_attention_fwd_static": (I, [S, P, P, P, P, P, P, F, P, P, P]),
        "psa_attention_bwd_workspace_bytes": (Z, [S]),
        "psa_quantize_qk_fp8": (I, [S, P, P, P, P, P, P, P, P, P]),
        "psa_attention_fp8_workspace_bytes": (Z, [S]),
        "psa_attention_fwd_fp8": (I, [S, P, P, P, P, P, P, F, P, P, P, Z, P]),
        "psa_attention_fwd_fp8_pv": (I, [S, P, P, P, P, P, P, F, P, P, P, Z, P]),
        "psa_attention_bwd": (I, [S, P, P, P, P, P, P, F, P, P, P, P, P, P, P, Z, P]),
        "psa_attention_plan_stats": (I, [S, P, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64), P]),
        "psa_get_device_status": (I, [P, P]),
        "psa_get_static_device_status": (I, [P]),
        "psa_debug_wait_control": (I, [P, ctypes.c_uint64, I, P]),
        "psa_last_error": (ctypes.c_char_p, []),
        "psa_version": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_LIB = None


def lib():
    """The loaded libpsa.so (loaded on first use; raises if it is not built)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


# ------------------------------------------------------------------------- marshalling

def _ptr(t: Optional[torch.Tensor], name: str, required: bool = True):
    if t is None:
        if required:
            raise ValueError("%s is required" % name)
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (the PSA path has no CPU fallback)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(st: int):
    if st != PSA_OK:
        raise PsaError(st, lib().psa_last_error().decode())


def make_shape(B, Hq, Hkv, N, d, block, levels, causal=False, dtype=PSA_DT_BF16) -> Shape:
    return Shape(B, Hq, Hkv, N, d, block, levels, int(bool(causal)), dtype)


def shape_of(q: torch.Tensor, k: torch.Tensor, block: int, levels: int, causal: bool = False) -> Shape:
    B, Hq, N, d = q.shape
    dt = PSA_DT_FP32 if q.dtype == torch.float32 else PSA_DT_BF16
    return make_shape(B, Hq, k.shape[1], N, d, block, levels, causal, dt)


def make_params(mode: int, thresholds: Sequence[float], sm_scale: float, stride: int = 8,
                cos_min: float = -3.0, n_dense_prefix: int = 0, n_samples: int = 8,
                policy: int = PSA_POLICY_MASS) -> MaskParams:
    th = (ctypes.c_float * 8)(*([float(t) for t in thresholds] + [0.0] * (8 - len(thresholds))))
    return MaskParams(mode, n_samples, stride, th, len(thresholds), cos_min, n_dense_prefix, sm_scale, policy)


def psa_version() -> int:
    return lib().psa_version()


def psa_last_error() -> str:
    return lib().psa_last_error().decode()


def psa_pyramid_bytes(shape: Shape) -> int:
    return lib().psa_pyramid_bytes(ctypes.byref(shape))


def psa_pyramid_level_offset(shape: Shape, level: int) -> int:
    return lib().psa_pyramid_level_offset(ctypes.byref(shape), level)


def psa_build_pyramid(shape: Shape, k, v, k_pyr, v_pyr, blockcos=None, stream=None):
    L1 = shape.levels > 1
    _check(lib().psa_build_pyramid(ctypes.byref(shape), _ptr(k, "k"), _ptr(v, "v"),
                                 _ptr(k_pyr, "k_pyr", L1), _ptr(v_pyr, "v_pyr", L1),
                                 _ptr(blockcos, "blockcos", False), _stream(stream)))


def psa_mask_workspace_bytes(shape: Shape, params: MaskParams) -> int:
    return lib().psa_mask_workspace_bytes(ctypes.byref(shape), ctypes.byref(params))


def psa_make_mask(shape: Shape, params: MaskParams, q, k, blockcos, mask, mass_out, workspace, stream=None):
    _check(lib().psa_make_mask(ctypes.byref(shape), ctypes.byref(params), _ptr(q, "q"), _ptr(k, "k"),
                             _ptr(blockcos, "blockcos", False), _ptr(mask, "mask"),
                             _ptr(mass_out, "mass_out", False), _ptr(workspace, "workspace"),
                             workspace.numel() * workspace.element_size(), _stream(stream)))


def psa_attention_workspace_bytes(shape: Shape) -> int:
    return lib().psa_attention_workspace_bytes(ctypes.byref(shape))


def psa_attention_fwd(shape: Shape, q, k, v, k_pyr, v_pyr, mask, sm_scale: float, out, lse, workspace,
                      stream=None):
    L1 = shape.levels > 1
    _check(lib().psa_attention_fwd(ctypes.byref(shape), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                 _ptr(k_pyr, "k_pyr", L1), _ptr(v_pyr, "v_pyr", L1), _ptr(mask, "mask"),
                                 ctypes.c_float(sm_scale), _ptr(out, "out"), _ptr(lse, "lse", False),
                                 _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                 _stream(stream)))


def psa_attention_fwd_static(shape: Shape, q, k, v, k_pyr, v_pyr, mask, sm_scale: float, out, lse, stream=None):
    """psa_attention_fwd on the library's own static device workspace (no
    workspace argument; for callers that cannot allocate device memory)."""
    L1 = shape.levels > 1
    _check(lib().psa_attention_fwd_static(ctypes.byref(shape), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                          _ptr(k_pyr, "k_pyr", L1), _ptr(v_pyr, "v_pyr", L1), _ptr(mask, "mask"),
                                          ctypes.c_float(sm_scale), _ptr(out, "out"), _ptr(lse, "lse", False),
                                          _stream(stream)))


def psa_quantize_qk_fp8(shape: Shape, q, k, k_pyr, q8, q_scale, k8, k8_pyr, k_scale, stream=None):
    L1 = shape.levels > 1
    _check(lib().psa_quantize_qk_fp8(ctypes.byref(shape), _ptr(q, "q"), _ptr(k, "k"), _ptr(k_pyr, "k_pyr", L1),
                                     _ptr(q8, "q8"), _ptr(q_scale, "q_scale"), _ptr(k8, "k8"),
                                     _ptr(k8_pyr, "k8_pyr", L1), _ptr(k_scale, "k_scale"), _stream(stream)))


def psa_attention_fp8_workspace_bytes(shape: Shape) -> int:
    return lib().psa_attention_fp8_workspace_bytes(ctypes.byref(shape))


def psa_attention_fwd_fp8(shape: Shape, q, k, v, k_pyr, v_pyr, mask, sm_scale: float, out, lse, workspace,
                          stream=None):
    L1 = shape.levels > 1
    _check(lib().psa_attention_fwd_fp8(ctypes.byref(shape), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                       _ptr(k_pyr, "k_pyr", L1), _ptr(v_pyr, "v_pyr", L1), _ptr(mask, "mask"),
                                       ctypes.c_float(sm_scale), _ptr(out, "out"), _ptr(lse, "lse", False),
                                       _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))


def psa_attention_fwd_fp8_pv(shape: Shape, q, k, v, k_pyr, v_pyr, mask, sm_scale: float, out, lse, workspace,
                             stream=None):
    L1 = shape.levels > 1
    _check(lib().psa_attention_fwd_fp8_pv(ctypes.byref(shape), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                          _ptr(k_pyr, "k_pyr", L1), _ptr(v_pyr, "v_pyr", L1), _ptr(mask, "mask"),
                                          ctypes.c_float(sm_scale), _ptr(out, "out"), _ptr(lse, "lse", False),
                                          _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                          _stream(stream)))


def psa_attention_bwd_workspace_bytes(shape: Shape) -> int:
    return lib().psa_attention_bwd_workspace_bytes(ctypes.byref(shape))


def psa_attention_bwd(shape: Shape, q, k, v, k_pyr, v_pyr, mask, sm_scale: float, out, lse, dout, dq, dk, dv,
                      workspace, stream=None):
    L1 = shape.levels > 1
    _check(lib().psa_attention_bwd(ctypes.byref(shape), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                   _ptr(k_pyr, "k_pyr", L1), _ptr(v_pyr, "v_pyr", L1), _ptr(mask, "mask"),
                                   ctypes.c_float(sm_scale), _ptr(out, "out"), _ptr(lse, "lse"), _ptr(dout, "dout"),
                                   _ptr(dq, "dq"), _ptr(dk, "dk"), _ptr(dv, "dv"), _ptr(workspace, "workspace"),
                                   ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))


def psa_attention_plan_stats(shape: Shape, workspace, stream=None):
    nt, nr = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(lib().psa_attention_plan_stats(ctypes.byref(shape), _ptr(workspace, "workspace"), ctypes.byref(nt),
                                        ctypes.byref(nr), _stream(stream)))
    return nt.value, nr.value


def psa_get_device_status(workspace, stream=None) -> int:
    return lib().psa_get_device_status(_ptr(workspace, "workspace"), _stream(stream))


def psa_get_static_device_status(stream=None) -> int:
    return lib().psa_get_static_device_status(_stream(stream))


def psa_debug_wait_control(workspace, limit_ns: int, trap: bool = False, stream=None):
    _check(lib().psa_debug_wait_control(_ptr(workspace, "workspace"), ctypes.c_uint64(limit_ns), int(bool(trap)),
                                        _stream(stream)))


# ------------------------------------------------------------------------- buffers

def pyramid_buffers(shape: Shape, device, dtype):
    """Uninitialised K/V pyramid buffers of the size the library asks for."""
    nb = psa_pyramid_bytes(shape)
    es = 4 if dtype == torch.float32 else 2
    n = max(nb // es, 1)
    return (torch.empty(n, dtype=dtype, device=device), torch.empty(n, dtype=dtype, device=device))


def pyramid_level(shape: Shape, buf: torch.Tensor, level: int) -> torch.Tensor:
    """View of level ``level`` (>= 1) inside a pyramid buffer: [B, Hkv, N/2^l, d]."""
    es = buf.element_size()
    off = psa_pyramid_level_offset(shape, level) // es
    n = shape.B * shape.Hkv * (shape.N >> level) * shape.d
    return buf[off:off + n].view(shape.B, shape.Hkv, shape.N >> level, shape.d)


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace (the status word must start at 0)."""
    n16 = max(1, (nbytes + 15) // 16)
    return torch.zeros(2 * n16, dtype=torch.int64, device=device).view(torch.uint8)[:max(nbytes, 16)]


# ------------------------------------------------------------------------- whole path

_CACHE = {}


def psa_forward(q, k, v, *, block: int = 128, levels: int = 4, thresholds: Sequence[float] = (0.6, 0.8, 0.9, 0.95),
                mode: int = PSA_MASK_SAMPLE, policy: int = PSA_POLICY_MASS, causal: bool = False,
                sm_scale: Optional[float] = None, stride: int = 8, cos_min: float = -3.0, n_dense_prefix: int = 0,
                mask=None, precision: str = "bf16", want_lse: bool = False, stream=None):
    """The whole forward path on device tensors: psa_build_pyramid (and the
    block cosines when cos_min > -2), psa_make_mask (unless a mask is given)
    and the attention (precision "bf16": psa_attention_fwd; "fp8":
    psa_attention_fwd_fp8; "fp8_pv": psa_attention_fwd_fp8_pv), on one
    stream.  q [B, Hq, N, d], k and v [B, Hkv, N, d], contiguous, bf16 (fp32
    for "bf16" only).  Pyramid buffers and workspaces are allocated on first
    use for a shape and reused.  Returns (out, mask, lse or None); a kernel
    time-out is reported by psa_forward_status()."""
    if precision not in ("bf16", "fp8", "fp8_pv"):
        raise ValueError("precision must be 'bf16', 'fp8' or 'fp8_pv', not %r" % (precision,))
    if len(thresholds) != levels:
        raise ValueError("%d thresholds for %d levels" % (len(thresholds), levels))
    shape = shape_of(q, k, block, levels, causal)
    scale = float(q.shape[-1]) ** -0.5 if sm_scale is None else float(sm_scale)
    params = make_params(mode, thresholds, scale, stride=stride, cos_min=cos_min, n_dense_prefix=n_dense_prefix,
                         policy=policy)
    key = (q.device, tuple(q.shape), tuple(k.shape), q.dtype, block, levels, causal, mode, stride, precision)
    c = _CACHE.get(key)
    if c is None:
        kp, vp = pyramid_buffers(shape, q.device, q.dtype)
        nb = -(-shape.N // block)
        attn_bytes = psa_attention_workspace_bytes(shape) if precision == "bf16" else \
            psa_attention_fp8_workspace_bytes(shape)
        c = {"kp": kp, "vp": vp,
             "bc": torch.empty(shape.B, shape.Hkv, nb, dtype=torch.float32, device=q.device),
             "mws": workspace(psa_mask_workspace_bytes(shape, params), q.device),
             "aws": workspace(attn_bytes, q.device)}
        _CACHE.clear()                        # one shape at a time: the buffers can be large
        _CACHE[key] = c
    bc = c["bc"] if cos_min > -2 else None
    L1 = levels > 1
    psa_build_pyramid(shape, k, v, c["kp"] if L1 else None, c["vp"] if L1 else None, bc, stream)
    if mask is None:
        nb = -(-shape.N // block)
        mask = torch.empty(shape.B, shape.Hq, nb, nb, dtype=torch.uint8, device=q.device)
        psa_make_mask(shape, params, q, k, bc, mask, None, c["mws"], stream)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    fn = {"bf16": psa_attention_fwd, "fp8": psa_attention_fwd_fp8, "fp8_pv": psa_attention_fwd_fp8_pv}[precision]
    fn(shape, q, k, v, c["kp"] if L1 else None, c["vp"] if L1 else None, mask, scale, out, lse, c["aws"], stream)
    return out, mask, lse


def psa_forward_status(stream=None) -> int:
    """Device status of the last psa_forward call (PSA_OK, or the first
    error of the mask or attention stage), read after the stream's work."""
    for c in _CACHE.values():
        for ws in (c["mws"], c["aws"]):
            st = psa_get_device_status(ws, stream)
            if st != PSA_OK:
                return st
    return PSA_OK
