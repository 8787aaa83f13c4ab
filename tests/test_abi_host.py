"""Host-only checks of the C ABI: the library loads, exports every function
include/psa.h declares, answers size queries, and rejects bad arguments with
the documented status before anything reaches a GPU (no device is used)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import video_transformers_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "psa.h")).read()
    return sorted(set(re.findall(r"PSA_API\s+[\w\s\*]+?\b(psa_\w+)\s*\(", src)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(P.EXPORTS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", P.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (psa_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(P.lib(), name) is not None


def test_version():
    assert P.psa_version() == 100


def test_pyramid_sizes():
    s = P.make_shape(1, 40, 40, 75600, 128, 128, 4)
    per_level = [1 * 40 * (75600 >> l) * 128 * 2 for l in (1, 2, 3)]
    assert P.psa_pyramid_bytes(s) == sum(per_level)
    assert P.psa_pyramid_level_offset(s, 1) == 0
    assert P.psa_pyramid_level_offset(s, 2) == per_level[0]
    assert P.psa_pyramid_level_offset(s, 3) == per_level[0] + per_level[1]
    assert P.psa_pyramid_level_offset(s, 4) == 0          # out of range
    s1 = P.make_shape(1, 2, 2, 1000, 64, 64, 1)
    assert P.psa_pyramid_bytes(s1) == 0
    sf = P.make_shape(1, 2, 2, 1024, 64, 64, 4, dtype=P.PSA_DT_FP32)
    assert P.psa_pyramid_bytes(sf) == 2 * (512 + 256 + 128) * 64 * 4
    for l in (2, 3):
        assert P.psa_pyramid_level_offset(sf, l) % 16 == 0


def test_workspace_sizes_positive_and_zero_on_bad_shape():
    s = P.make_shape(1, 28, 4, 32768, 128, 128, 4, causal=True)
    p = P.make_params(P.PSA_MASK_ANTIDIAG, (0.9, 0.95, 0.975, 0.9875), 128 ** -0.5, stride=8, cos_min=0.8)
    assert P.psa_mask_workspace_bytes(s, p) > 28 * 4096 * 256 * 4
    assert P.psa_attention_workspace_bytes(s) > 0
    bad = P.make_shape(1, 28, 4, 32768, 96, 128, 4)
    assert P.psa_attention_workspace_bytes(bad) == 0
    assert P.psa_mask_workspace_bytes(bad, p) == 0


FAKE = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced: every case fails validation first
MIS = ctypes.c_void_p((1 << 20) + 8)


def _attn(shape, q=FAKE, k=FAKE, v=FAKE, kp=FAKE, vp=FAKE, mask=FAKE, scale=0.1, out=FAKE, lse=None,
          ws=FAKE, ws_bytes=1 << 40):
    return P.lib().psa_attention_fwd(ctypes.byref(shape), q, k, v, kp, vp, mask, ctypes.c_float(scale), out, lse,
                                     ws, ws_bytes, None)


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, P.PSA_ERR_UNSUPPORTED),
    ("d", 0, P.PSA_ERR_INVALID_ARG),
    ("block", 32, P.PSA_ERR_UNSUPPORTED),
    ("levels", 5, P.PSA_ERR_UNSUPPORTED),
    ("levels", 0, P.PSA_ERR_INVALID_ARG),
    ("N", 1001, P.PSA_ERR_UNSUPPORTED),      # not a multiple of 2^(L-1) = 8
    ("Hkv", 3, P.PSA_ERR_UNSUPPORTED),       # 4 % 3 != 0
    ("dtype", 7, P.PSA_ERR_INVALID_ARG),
    ("B", -1, P.PSA_ERR_INVALID_ARG),
    ("B", 0, P.PSA_ERR_INVALID_ARG),         # empty inputs are rejected, nothing is written
    ("Hq", 0, P.PSA_ERR_INVALID_ARG),
    ("N", 0, P.PSA_ERR_INVALID_ARG),
])
def test_attention_rejects_bad_shape(field, value, code):
    s = P.make_shape(1, 4, 2, 1000 if field != "N" else 1000, 64, 64, 4)
    s.N = 1024
    setattr(s, field, value)
    assert _attn(s) == code
    assert P.psa_last_error() != ""


def test_attention_rejects_bad_pointers_and_workspace():
    s = P.make_shape(1, 4, 2, 1024, 64, 64, 4)
    assert _attn(s, q=None) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, out=None) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, mask=None) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, kp=None) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, k=MIS) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, lse=MIS) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, scale=0.0) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, scale=float("nan")) == P.PSA_ERR_INVALID_ARG
    assert _attn(s, ws=None) == P.PSA_ERR_WORKSPACE
    assert _attn(s, ws_bytes=P.psa_attention_workspace_bytes(s) - 1) == P.PSA_ERR_WORKSPACE
    assert "workspace" in P.psa_last_error()
    s1 = P.make_shape(1, 4, 2, 1024, 64, 64, 1)    # L = 1: pyramid pointers may be NULL ...
    assert _attn(s1, kp=None, vp=None, ws=None) == P.PSA_ERR_WORKSPACE   # ... and validation goes on


def test_pyramid_rejects_bad_args():
    s = P.make_shape(1, 2, 2, 1024, 64, 64, 4)
    lib = P.lib()
    assert lib.psa_build_pyramid(ctypes.byref(s), None, FAKE, FAKE, FAKE, None, None) == P.PSA_ERR_INVALID_ARG
    assert lib.psa_build_pyramid(ctypes.byref(s), FAKE, FAKE, None, FAKE, None, None) == P.PSA_ERR_INVALID_ARG
    assert lib.psa_build_pyramid(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, MIS, None) == P.PSA_ERR_INVALID_ARG
    s.N = 1020
    assert lib.psa_build_pyramid(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, None) == P.PSA_ERR_UNSUPPORTED
    assert lib.psa_build_pyramid(None, FAKE, FAKE, FAKE, FAKE, None, None) == P.PSA_ERR_INVALID_ARG


def test_mask_rejects_bad_params():
    s = P.make_shape(1, 4, 2, 1024, 64, 64, 4)
    lib = P.lib()

    def call(p, blockcos=None, ws_bytes=1 << 40, mask=FAKE):
        return lib.psa_make_mask(ctypes.byref(s), ctypes.byref(p), FAKE, FAKE, blockcos, mask, None, FAKE,
                                 ws_bytes, None)
    good = P.make_params(P.PSA_MASK_SAMPLE, (0.6, 0.8, 0.9, 0.95), 0.125)
    assert call(P.make_params(P.PSA_MASK_SAMPLE, (0.6, 0.8, 0.9), 0.125)) == P.PSA_ERR_INVALID_ARG
    assert call(P.make_params(P.PSA_MASK_SAMPLE, (0.6, 0.8, 0.9, 0.95), 0.125, n_samples=4)) == P.PSA_ERR_UNSUPPORTED
    assert call(P.make_params(P.PSA_MASK_ANTIDIAG, (0.6, 0.8, 0.9, 0.95), 0.125, stride=3)) == P.PSA_ERR_UNSUPPORTED
    assert call(P.make_params(P.PSA_MASK_ANTIDIAG, (0.6, 0.8, 0.9, 0.95), 0.125, stride=16)) == P.PSA_ERR_UNSUPPORTED
    assert call(P.make_params(7, (0.6, 0.8, 0.9, 0.95), 0.125)) == P.PSA_ERR_INVALID_ARG
    assert call(P.make_params(P.PSA_MASK_SAMPLE, (0.6, 0.8, 0.9, 0.95), 0.125, cos_min=0.8)) == P.PSA_ERR_INVALID_ARG
    assert call(good, mask=None) == P.PSA_ERR_INVALID_ARG
    assert call(good, ws_bytes=16) == P.PSA_ERR_WORKSPACE
    assert call(P.make_params(P.PSA_MASK_SAMPLE, (0.6, 0.8, 0.9, 0.95), 0.125, policy=2)) == P.PSA_ERR_INVALID_ARG
    assert call(P.make_params(3, (0.6, 0.8, 0.9, 0.95), 0.125)) == P.PSA_ERR_INVALID_ARG
    mk = P.make_params(P.PSA_MASK_MEANKEY, (0.6, 0.8, 0.9, 0.95), 0.125, policy=P.PSA_POLICY_QUANTILE)
    assert call(mk, ws_bytes=16) == P.PSA_ERR_WORKSPACE


def test_meankey_workspace_needs_no_alignment():
    """The mean-key scorer takes any N (sampling needs N % (block/8) == 0);
    its workspace holds the score rows and the fp64 block means."""
    s = P.make_shape(2, 4, 2, 1001, 128, 64, 1)       # one level: a binary mask, any N
    nb = -(-1001 // 64)
    samp = P.make_params(P.PSA_MASK_SAMPLE, (0.9,), 0.1)
    mk = P.make_params(P.PSA_MASK_MEANKEY, (0.9,), 0.1)
    assert P.psa_mask_workspace_bytes(s, samp) == 0
    need = P.psa_mask_workspace_bytes(s, mk)
    floor = 2 * 4 * nb * nb * 4 + 2 * 2 * 4 * nb * 4 + 2 * 4 * nb * 128 * 8 + 2 * 2 * nb * 128 * 8
    assert floor <= need <= floor + 8 * 256 + 256


def test_struct_layouts_match_the_header(tmp_path):
    """sizeof / offsetof of the two parameter structs, from gcc compiling the
    public header, against the ctypes binding."""
    prog = tmp_path / "layout.c"
    fields_s = [f for f, _ in P.Shape._fields_]
    fields_m = [f for f, _ in P.MaskParams._fields_]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "psa.h"', 'int main(void) {',
             '  printf("%zu\\n", sizeof(psa_shape_t));', '  printf("%zu\\n", sizeof(psa_mask_params_t));']
    lines += ['  printf("%%zu\\n", offsetof(psa_shape_t, %s));' % f for f in fields_s]
    lines += ['  printf("%%zu\\n", offsetof(psa_mask_params_t, %s));' % f for f in fields_m]
    lines += ['  return 0;', '}']
    prog.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [ctypes.sizeof(P.Shape), ctypes.sizeof(P.MaskParams)]
    want += [getattr(P.Shape, f).offset for f in fields_s] + [getattr(P.MaskParams, f).offset for f in fields_m]
    assert got == want


def test_binding_refuses_cpu_tensors():
    import torch
    s = P.make_shape(1, 2, 2, 64, 64, 64, 1)
    k = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        P.psa_build_pyramid(s, k, k, None, None)


def test_debug_wait_control_rejects_null_and_misaligned():
    assert P.lib().psa_debug_wait_control(None, 5, 1, None) == P.PSA_ERR_INVALID_ARG
    assert P.lib().psa_debug_wait_control(ctypes.c_void_p(0x1003), 5, 0, None) == P.PSA_ERR_INVALID_ARG
    assert "workspace" in P.psa_last_error()


def test_fp8_path_rejects_unsupported_shapes():
    s64 = P.make_shape(1, 2, 2, 256, 64, 64, 4)
    assert P.psa_attention_fp8_workspace_bytes(s64) == 0
    x = torch.empty(16, dtype=torch.uint8)
    st = P.lib().psa_attention_fwd_fp8(ctypes.byref(s64), *([ctypes.c_void_p(16)] * 6), ctypes.c_float(0.1),
                                       ctypes.c_void_p(16), None, ctypes.c_void_p(16), 1 << 30, None)
    assert st == P.PSA_ERR_UNSUPPORTED and "128" in P.psa_last_error()
    st = P.lib().psa_attention_fwd_fp8_pv(ctypes.byref(s64), *([ctypes.c_void_p(16)] * 6), ctypes.c_float(0.1),
                                          ctypes.c_void_p(16), None, ctypes.c_void_p(16), 1 << 30, None)
    assert st == P.PSA_ERR_UNSUPPORTED and "128" in P.psa_last_error()
    sf = P.make_shape(1, 2, 2, 256, 128, 64, 4, dtype=P.PSA_DT_FP32)
    assert P.psa_attention_fp8_workspace_bytes(sf) == 0
    assert P.psa_attention_fp8_workspace_bytes(P.make_shape(1, 2, 2, 256, 128, 64, 4)) > 0


def test_psa_forward_rejects_bad_arguments():
    """The whole-path convenience call checks its options before any launch."""
    x = torch.zeros(1, 1, 128, 64)
    with pytest.raises(ValueError):
        P.psa_forward(x, x, x, precision="int4")
    with pytest.raises(ValueError):
        P.psa_forward(x, x, x, levels=4, thresholds=(0.5, 0.9))
