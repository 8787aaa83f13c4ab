"""Seeded synthetic inputs for the PSA forward path.

This module is shared by the tests, the benchmark and the smoke check.  It
holds the workload presets and the random-input recipes only: none of the
method's arithmetic (pooling, scoring, level assignment, attention) lives
here, so both the CUDA path and the CPU oracle can draw their inputs from it
without sharing any of the computation they are compared on.

Recipes
-------
* ``iid``: every element ~ N(0, 1).
* ``field``: per (tensor, head, channel), an independent N(0, 1) grid over the
  video latent (T, H, W), low-pass filtered by a Gaussian whose correlation
  function is exp(-r^2 / (2 * 4^2)) (kernel sigma = 4 / sqrt(2) per axis,
  FFT, periodic boundaries), standardised to mean 0 / std 1 per channel,
  plus 0.3 * N(0, 1) noise.  Tokens are flattened frame-major (t, then h,
  then w).  Text tokens, where a preset has them, come first and are iid.

The presets mirror the five workload shapes the method is evaluated on:
a tiny fp32 case, Wan2.1-1.3B and Wan2.1-14B shaped self-attention,
CogVideoX-5B shaped joint text+video attention, and Qwen2.5-VL-7B shaped
causal GQA prefill.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional, Sequence, Tuple

import torch

SKIP = 0xFF


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    block: int
    levels: int
    causal: bool
    dtype: str                      # "fp32" or "bf16"
    recipe: str                     # "iid" or "field"
    grid: Tuple[int, int, int] = (0, 0, 0)   # (T, H, W) of the video latent
    n_text: int = 0                 # iid text tokens placed before the video tokens
    n_iid: int = 0                  # total tokens for the iid recipe
    mask_mode: str = "given"        # "given" (drawn here), "sample", "antidiag" or "meankey"
    thresholds: Tuple[float, ...] = ()
    policy: str = "mass"            # level policy: "mass" (thresholds on the mass prefix) or "quantile"
    n_samples: int = 8
    stride: int = 8
    cos_min: float = -3.0           # <= -2 disables the cosine gate
    n_dense_prefix: int = 0
    seed: int = 0

    @property
    def N(self) -> int:
        if self.recipe == "iid":
            return self.n_iid
        T, H, W = self.grid
        return self.n_text + T * H * W

    @property
    def nqb(self) -> int:
        return -(-self.N // self.block)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def antidiag_thresholds(t0: float, levels: int) -> Tuple[float, ...]:
    """Thresholds for the understanding preset, which names a single cut t0.

    The keep set of a binary mask at t0 becomes level 0; the residual mass
    above it is halved per further level: t_l = 1 - (1 - t0) * 2^-l.
    """
    return tuple(1.0 - (1.0 - t0) * 2.0 ** (-l) for l in range(levels))


PRESETS = {
    "tiny": Workload("tiny", B=1, Hq=2, Hkv=2, d=64, block=64, levels=4, causal=False,
                     dtype="fp32", recipe="iid", n_iid=1024, mask_mode="given", seed=0),
    "wan1.3b": Workload("wan1.3b", B=1, Hq=12, Hkv=12, d=128, block=64, levels=4, causal=False,
                        dtype="bf16", recipe="field", grid=(21, 30, 52), mask_mode="sample",
                        thresholds=(0.6, 0.8, 0.9, 0.95), seed=1),
    "cogvideox5b": Workload("cogvideox5b", B=1, Hq=48, Hkv=48, d=64, block=64, levels=4,
                            causal=False, dtype="bf16", recipe="field", grid=(13, 30, 45),
                            n_text=226, mask_mode="sample", thresholds=(0.5, 0.7, 0.85, 0.9),
                            n_dense_prefix=226, seed=2),
    "qwen2.5vl": Workload("qwen2.5vl", B=1, Hq=28, Hkv=4, d=128, block=128, levels=4, causal=True,
                          dtype="bf16", recipe="field", grid=(64, 16, 32), mask_mode="antidiag",
                          thresholds=antidiag_thresholds(0.9, 4), stride=8, cos_min=0.8, seed=3),
    "wan14b": Workload("wan14b", B=1, Hq=40, Hkv=40, d=128, block=128, levels=4, causal=False,
                       dtype="bf16", recipe="field", grid=(21, 45, 80), mask_mode="sample",
                       thresholds=(0.6, 0.8, 0.9, 0.95), seed=4),
}
ORDER = ["tiny", "wan1.3b", "cogvideox5b", "qwen2.5vl", "wan14b"]


def reduced(name: str, grid: Optional[Tuple[int, int, int]] = None, heads: Optional[Tuple[int, int]] = None,
            n_text: Optional[int] = None, n_iid: Optional[int] = None) -> Workload:
    """A smaller copy of a preset with the same structure (block, levels,
    mask mode, causal flag, GQA ratio, text prefix), for cases the oracle
    finishes in seconds."""
    w = PRESETS[name]
    kw = {"name": name + "-reduced"}
    if grid is not None:
        kw["grid"] = grid
    if heads is not None:
        kw["Hq"], kw["Hkv"] = heads
    if n_text is not None:
        kw["n_text"] = n_text
        kw["n_dense_prefix"] = n_text if w.n_dense_prefix else 0
    if n_iid is not None:
        kw["n_iid"] = n_iid
    return w.replace(**kw)


# --------------------------------------------------------------------------------------
# random recipes
# --------------------------------------------------------------------------------------

def _gaussian_transfer(grid, corr_len: float, device) -> torch.Tensor:
    """Fourier-domain transfer function of a separable Gaussian filter with
    sigma = corr_len / sqrt(2) per axis (periodic boundaries)."""
    sigma = corr_len / math.sqrt(2.0)
    T, H, W = grid
    ft = torch.fft.fftfreq(T, device=device, dtype=torch.float64)
    fh = torch.fft.fftfreq(H, device=device, dtype=torch.float64)
    fw = torch.fft.rfftfreq(W, device=device, dtype=torch.float64)
    f2 = ft[:, None, None] ** 2 + fh[None, :, None] ** 2 + fw[None, None, :] ** 2
    return torch.exp(-2.0 * math.pi ** 2 * sigma ** 2 * f2).to(torch.float32)


def smooth_field(n_fields: int, grid, gen: torch.Generator, device, corr_len: float = 4.0,
                 noise: float = 0.3, chunk: int = 512) -> torch.Tensor:
    """``n_fields`` independent smoothed fields, returned as [n_fields, T*H*W]
    float32 (frame-major flattening)."""
    T, H, W = grid
    tf = _gaussian_transfer(grid, corr_len, device)
    out = torch.empty(n_fields, T * H * W, dtype=torch.float32, device=device)
    for c0 in range(0, n_fields, chunk):
        c1 = min(n_fields, c0 + chunk)
        white = torch.randn(c1 - c0, T, H, W, generator=gen, device=device, dtype=torch.float32)
        f = torch.fft.irfftn(torch.fft.rfftn(white, dim=(1, 2, 3)) * tf, s=(T, H, W), dim=(1, 2, 3))
        f = f.reshape(c1 - c0, -1)
        f = (f - f.mean(dim=1, keepdim=True)) / f.std(dim=1, keepdim=True)
        f = f + noise * torch.randn(f.shape, generator=gen, device=device, dtype=torch.float32)
        out[c0:c1] = f
    return out


def _field_tensor(w: Workload, H: int, gen, device) -> torch.Tensor:
    """[B, H, N, d] float32 following the ``field`` recipe."""
    T, GH, GW = w.grid
    nv = T * GH * GW
    x = torch.empty(w.B, H, w.N, w.d, dtype=torch.float32, device=device)
    for b in range(w.B):
        for h in range(H):
            if w.n_text:
                x[b, h, :w.n_text] = torch.randn(w.n_text, w.d, generator=gen, device=device)
            f = smooth_field(w.d, w.grid, gen, device)          # [d, nv]
            x[b, h, w.n_text:] = f.t()
    return x


def _new_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_qkv(w: Workload, device="cpu", seed: Optional[int] = None):
    """Q [B,Hq,N,d], K/V [B,Hkv,N,d] in the preset's dtype on ``device``.

    Draw order: Q, K, V (then, for the tiny preset, the mask; see
    :func:`make_given_mask`)."""
    gen = _new_gen(w.seed if seed is None else seed, device)
    if w.recipe == "iid":
        q = torch.randn(w.B, w.Hq, w.N, w.d, generator=gen, device=device)
        k = torch.randn(w.B, w.Hkv, w.N, w.d, generator=gen, device=device)
        v = torch.randn(w.B, w.Hkv, w.N, w.d, generator=gen, device=device)
    else:
        q = _field_tensor(w, w.Hq, gen, device)
        k = _field_tensor(w, w.Hkv, gen, device)
        v = _field_tensor(w, w.Hkv, gen, device)
    dt = w.torch_dtype
    return q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(), gen


def make_given_mask(w: Workload, gen: torch.Generator, device="cpu", p_skip: float = 0.2,
                    causal_diag: bool = True) -> torch.Tensor:
    """A mask drawn pair by pair: level 0..L-1 or SKIP with equal
    probability (for L=4: 0.2 each), diagonal forced to level 0.  Returns
    uint8 [B, Hq, nQB, nKB]."""
    nb = w.nqb
    m = torch.randint(0, w.levels + 1, (w.B, w.Hq, nb, nb), generator=gen, device=device)
    m = torch.where(m == w.levels, torch.full_like(m, SKIP), m).to(torch.uint8)
    if causal_diag:
        idx = torch.arange(nb, device=device)
        m[:, :, idx, idx] = 0
    if w.causal:
        upper = torch.triu(torch.ones(nb, nb, dtype=torch.bool, device=device), diagonal=1)
        m[:, :, upper] = SKIP
    return m


def random_mask(B, H, nqb, nkb, levels, gen, device="cpu", p_skip=None) -> torch.Tensor:
    """Uniform mask over {0..L-1, SKIP} with no forced structure (for edge-case tests)."""
    m = torch.randint(0, levels + 1, (B, H, nqb, nkb), generator=gen, device=device)
    return torch.where(m == levels, torch.full_like(m, SKIP), m).to(torch.uint8)


def sha256(t: torch.Tensor) -> str:
    return hashlib.sha256(t.detach().cpu().contiguous().view(torch.uint8).numpy().tobytes()).hexdigest()


def dense_flops(w: Workload) -> float:
    """FLOPs of dense (all level 0) attention: 4 * d * N^2 per (b, h)."""
    return 4.0 * w.d * w.N * w.N * w.B * w.Hq
