"""psa_attention_fwd_static: attention without a caller-provided workspace.

Some callers cannot allocate device memory themselves (a plugin inside a host
framework that owns every device allocation, or a latency-critical loop that
cannot afford cudaMalloc's implicit synchronisation).  This entry point runs
on a fixed device array inside libpsa.so instead.  The test calls it through
the C ABI twice in a row, on two different problems (so the second call
starts from the first call's leftovers in the shared array), compares each
output bit for bit with psa_attention_fwd on an allocated workspace, and
reads the array's status word after each call.  This file is collected last
on purpose."""
import ctypes

import pytest
import torch

import video_transformers_b200 as P
from psa_run import SKIP, run_attention, run_pyramid

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _problem(seed, B, Hq, Hkv, N, d, block, L, causal):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, N, d, generator=g).bfloat16().to(DEV)
    k = torch.randn(B, Hkv, N, d, generator=g).bfloat16().to(DEV)
    v = torch.randn(B, Hkv, N, d, generator=g).bfloat16().to(DEV)
    nb = -(-N // block)
    m = torch.randint(0, L + 1, (B, Hq, nb, nb), generator=g)
    mask = torch.where(m == L, torch.full_like(m, SKIP), m).to(torch.uint8).to(DEV)
    shape = P.make_shape(B, Hq, Hkv, N, d, block, L, causal)
    return shape, q, k, v, mask


def test_static_workspace_matches_allocating_entry_point():
    """Both entry points run the same plan and kernels on the same inputs,
    and the kernels are deterministic (the order of work inside a query
    tile does not depend on which CTA takes it), so the outputs must be
    identical bit for bit.  The second static call runs on the leftovers of
    the first in the shared array.  No call may change the device's free
    memory once the library's modules are loaded, and the static array's
    status word must read PSA_OK after each call."""
    problems = [(1, 2, 8, 4, 1000, 128, 128, 4, False), (2, 1, 4, 2, 900, 64, 64, 3, True)]
    for i, p in enumerate(problems):
        shape, q, k, v, mask = _problem(*p)
        assert P.psa_attention_workspace_bytes(shape) <= (32 << 20)
        kp, vp, _ = run_pyramid(shape, k, v)
        ref, ref_lse, _ = run_attention(shape, q, k, v, kp, vp, mask, shape.d ** -0.5)
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=DEV)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        P.psa_attention_fwd_static(shape, q, k, v, kp, vp, mask, shape.d ** -0.5, out, lse)
        assert P.psa_get_static_device_status() == P.PSA_OK, P.psa_last_error()
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        if i > 0:
            assert free1 == free0, (free0, free1)
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)
        err = (out.float() - ref.float()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


def test_static_workspace_rejects_oversized_shape():
    shape = P.make_shape(1, 40, 40, 75600, 128, 128, 4)     # needs far more than 32 MiB of plan
    assert P.psa_attention_workspace_bytes(shape) > (32 << 20)
    x = torch.empty(16, dtype=torch.uint8, device=DEV)
    st = P.lib().psa_attention_fwd_static(ctypes.byref(shape), *([ctypes.c_void_p(x.data_ptr())] * 6),
                                          ctypes.c_float(0.1), ctypes.c_void_p(x.data_ptr()), None, None)
    assert st == P.PSA_ERR_WORKSPACE
    assert "static workspace" in P.psa_last_error()
