#!/usr/bin/env python3
"""Benchmark of the PSA forward path (pyramid -> mask -> attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config wan14b] [--impl psa|reference]

One step = one pass of the whole path over one synthetic input of the
chosen workload (default: the Wan2.1-14B-shaped 720p self-attention, B1 H40
N75600 d128 bf16, block 128, L 4, sampling mask): psa_build_pyramid,
psa_make_mask, psa_attention_fwd, all through the C ABI.  Inputs (2.3 GB)
are larger than L2, so no flush is needed between steps.

value = executed attention FLOPs of all ranks / (max over ranks of the
device time of K steps) in TFLOP/s, where executed FLOPs count only real
work: 4 d sum over (b, h, I) of (query rows of I) x (pooled key rows the
mask fetches for I); skipped blocks and tile padding are not work.

--impl reference times the CPU oracle (the only other implementation of
this path) on the machine's host cores, on a bounded sample of the same
workload, in the same unit.  With torchrun (N > 1) every rank runs its own
full workload instance (weak scaling, no data-path collective); only the
timing is reduced (max over ranks).  --split heads instead splits one
problem's heads over the ranks (strong scaling), with the all-gather of the
output timed apart.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "PSA attn fwd ms/call & achieved TFLOP/s (executed FLOPs) vs B200 BF16 peak"
# DRAM traffic of one attention launch (dram__bytes_read.sum + dram__bytes_write.sum), from an
# ncu capture of the same workload at 4 heads scaled to the full head count (traffic grows with
# the heads: the head-major queue keeps one head's KV in L2 at a time); valid only for the
# attention source it was measured on, identified by its SHA-256.
ATTN_TRAFFIC = {"wan14b": {"bytes_per_launch": 10 * (824.550144e6 + 72.312576e6),
                           "attn_cu_sha256": "9465fd8804337046dccd787be24237362f6a682c1dc5d59b6e3b479e6c61bdb2"}}
UNIT = "TFLOP/s"
KERNELS_PER_STEP = {"pyramid": 1, "blockcos": 0, "score": 1, "select": 1, "plan": 3, "attention": 1}
# kernels of psa_make_mask per scorer: score + select, or block means (Q, K),
# logits, row LSE + select; a given mask is a device copy, none of ours
MASK_KERNELS = {"sample": 2, "antidiag": 2, "meankey": 5, "given": 0}
MUFU_PER_CLK_SM = 16       # ex2.approx.ftz.f32 per clock per SM (measured on B200)


def mask_roofline(w, mask_ms, hbm, clocks, elem):
    """Roofline of the whole mask stage (scorer + select): the sampling and
    antidiagonal scorers are bound by one exp2 per score element on the
    special-function unit; the mean-key scorer by reading Q and K once."""
    if w.mask_mode == "meankey":
        byts = w.B * (w.Hq + w.Hkv) * w.N * w.d * elem
        ach = byts / (mask_ms * 1e-3) / 1e9
        return {"bound": "hbm", "stage": "psa_make_mask", "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": ach / hbm, "work": "Q and K read once, %.3f GB" % (byts / 1e9)}
    if w.mask_mode not in ("sample", "antidiag"):
        return None
    if w.mask_mode == "sample":
        rows, cols = -(-w.N // w.block) * 8, w.N
    else:
        rows = cols = w.N // w.stride
    exps = rows * cols * w.B * w.Hq * (0.5 if w.causal else 1.0)
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = MUFU_PER_CLK_SM * 148 * mhz * 1e6 / 1e9
    ach = exps / (mask_ms * 1e-3) / 1e9
    return {"bound": "alu", "unit_kind": "special-function unit (exp2)", "stage": "psa_make_mask",
            "achieved": ach, "peak": peak, "unit": "Gexp2/s", "frac": ach / peak,
            "work": "%.3g exp2 (one per score element); peak = %d/clk/SM x 148 SMs x %.0f MHz (sampled clock)"
                    % (exps, MUFU_PER_CLK_SM, mhz)}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers

def attn_traffic(w):
    """Measured DRAM bytes per attention launch for this workload, or None when
    there is no capture of it or the attention source changed since."""
    import hashlib
    rec = ATTN_TRAFFIC.get(w.name)
    if rec is None:
        return None
    with open(os.path.join(ROOT, "video_transformers_b200", "csrc", "attn.cu"), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["attn_cu_sha256"]:
            return None
    return rec["bytes_per_launch"]


def max_over_ranks(ms: float, world: int, device) -> float:
    """Device time of the timed region, max over ranks (every rank takes
    this collective at the same point)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def head_partition(Hq: int, Hkv: int, rank: int, world: int):
    """The KV heads [hkv0, hkv1) and query heads [hq0, hq1) of one rank when
    the heads of one problem are split over `world` GPUs: KV heads in equal
    contiguous runs, each with the query heads that read it (GQA groups are
    never split).  Needs Hkv % world == 0."""
    if Hkv % world:
        raise ValueError("Hkv = %d is not a multiple of %d GPUs" % (Hkv, world))
    per = Hkv // world
    grp = Hq // Hkv
    hkv0, hkv1 = rank * per, (rank + 1) * per
    return hkv0 * grp, hkv1 * grp, hkv0, hkv1


def gather_heads(x: torch.Tensor, world: int) -> torch.Tensor:
    """All-gather of a [B, H_local, ...] tensor along the head axis: the full
    output on every rank (NCCL over NVLink on GPUs; any backend works)."""
    if world <= 1:
        return x
    parts = [torch.empty_like(x) for _ in range(world)]
    torch.distributed.all_gather(parts, x.contiguous())
    return torch.cat(parts, dim=1)


def aggregate_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank runs its own workload instance of
    `flops_per_rank` executed FLOPs per step (weak scaling)."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def executed_flops(mask: torch.Tensor, N: int, block: int, d: int, levels: int, causal: bool) -> float:
    """4 d sum_{b,h,I} q_I * sum_{J: M != SKIP} k_J / 2^l (on the device)."""
    dev = mask.device
    nb = mask.shape[-1]
    idx = torch.arange(nb, device=dev)
    qrows = (torch.clamp((idx + 1) * block, max=N) - idx * block).double()
    m = mask.long()
    total = torch.zeros((), dtype=torch.float64, device=dev)
    for l in range(levels):
        krows = ((torch.clamp((idx + 1) * block, max=N) - idx * block) // (1 << l)).double()
        sel = (m == l).double()
        if causal:
            sel = sel * torch.tril(torch.ones(nb, nb, device=dev, dtype=torch.float64))
        total += (sel * qrows[:, None] * krows[None, :]).sum()
    return 4.0 * d * float(total.item())


def diagonal_excess_flops(mask: torch.Tensor, N: int, block: int, d: int) -> float:
    """FLOPs that executed_flops counts for the key-after-query pairs of the
    causal diagonal blocks (always level 0): q_I^2 - q_I (q_I + 1) / 2 per
    (b, h, I) whose diagonal is not skipped.  Subtracting them gives the
    FlashAttention convention, where a causal block counts only its visible
    pairs."""
    dev = mask.device
    nb = mask.shape[-1]
    idx = torch.arange(nb, device=dev)
    qrows = (torch.clamp((idx + 1) * block, max=N) - idx * block).double()
    diag = (mask.diagonal(dim1=-2, dim2=-1) == 0).double()
    return 4.0 * d * float((diag * (qrows * qrows - qrows * (qrows + 1) / 2)).sum().item())


class Path:
    """Device buffers and the three ABI calls of one workload instance."""

    def __init__(self, w: W.Workload, q, k, v):
        import video_transformers_b200 as P
        self.P, self.w = P, w
        self.q, self.k, self.v = q, k, v
        dev = q.device
        self.shape = P.make_shape(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.levels, w.causal,
                                  P.PSA_DT_FP32 if w.dtype == "fp32" else P.PSA_DT_BF16)
        mode = {"sample": P.PSA_MASK_SAMPLE, "meankey": P.PSA_MASK_MEANKEY}.get(w.mask_mode, P.PSA_MASK_ANTIDIAG)
        policy = P.PSA_POLICY_QUANTILE if w.policy == "quantile" else P.PSA_POLICY_MASS
        self.params = P.make_params(mode, w.thresholds or (0.6, 0.8, 0.9, 0.95)[:w.levels], w.sm_scale,
                                    stride=w.stride, cos_min=w.cos_min, n_dense_prefix=w.n_dense_prefix,
                                    policy=policy)
        self.kp, self.vp = P.pyramid_buffers(self.shape, dev, q.dtype)
        nb = w.nqb
        self.bc = torch.empty(w.B, w.Hkv, nb, dtype=torch.float32, device=dev) if w.cos_min > -2 else None
        self.mask = torch.empty(w.B, w.Hq, nb, nb, dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(q)
        self.mws = P.workspace(P.psa_mask_workspace_bytes(self.shape, self.params), dev)
        self.aws = P.workspace(P.psa_attention_workspace_bytes(self.shape), dev)
        self.given_mask = None
        self.stream = None          # torch stream the ABI calls are enqueued on (None: the current one)

    def _s(self):
        return None if self.stream is None else self.stream.cuda_stream

    def pyramid(self):
        self.P.psa_build_pyramid(self.shape, self.k, self.v, self.kp, self.vp, self.bc, self._s())

    def make_mask(self):
        if self.given_mask is not None:
            self.mask.copy_(self.given_mask)
        else:
            self.P.psa_make_mask(self.shape, self.params, self.q, self.k, self.bc, self.mask, None, self.mws,
                                 self._s())

    def attention(self, mask=None):
        self.P.psa_attention_fwd(self.shape, self.q, self.k, self.v, self.kp, self.vp,
                                 self.mask if mask is None else mask, self.w.sm_scale, self.out, None, self.aws,
                                 self._s())

    def step(self):
        self.pyramid()
        self.make_mask()
        self.attention()


# ----------------------------------------------------------------------------- psa arm

T0 = time.time()


def log(args, msg):
    if args.verbose:
        sys.stderr.write("[bench %7.2fs] %s\n" % (time.time() - T0, msg))
        sys.stderr.flush()


TENSOR_FLOP_PER_CLK_SM = 8192     # dense bf16 tcgen05 rate per SM per clock (M128 N256 K16 in 128 cycles)


def measure(path, w, args, steps, warmup, stream, world=1, dev=None, dense=True):
    """Warm-up, then `steps` timed steps with events around each stage;
    returns the stage times, executed flops, plan stats and the dense
    (all-level-0) attention time."""
    P = path.P
    for _ in range(warmup):
        path.step()
    torch.cuda.synchronize()
    flops = executed_flops(path.mask, w.N, w.block, w.d, w.levels, w.causal)
    n_tiles, n_rows = P.psa_attention_plan_stats(path.shape, path.aws)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        path.pyramid()
        ev[i][1].record(stream)
        path.make_mask()
        ev[i][2].record(stream)
        path.attention()
        ev[i][3].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    total_ms = max_over_ranks(start.elapsed_time(stop), world, dev)
    st = P.psa_get_device_status(path.aws) or P.psa_get_device_status(path.mws)
    if st != P.PSA_OK:
        raise RuntimeError("device status %d after the timed region: %s" % (st, P.psa_last_error()))
    r = {"total_ms": total_ms, "flops": flops, "n_tiles": n_tiles, "n_rows": n_rows,
         "pyr_ms": statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps)),
         "mask_ms": statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(steps)),
         "attn_ms": statistics.mean(ev[i][2].elapsed_time(ev[i][3]) for i in range(steps)),
         "dense_ms": None}
    if dense:
        dense_mask = torch.zeros_like(path.mask)
        path.attention(dense_mask)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 2
        e0.record(stream)
        for _ in range(reps):
            path.attention(dense_mask)
        e1.record(stream)
        torch.cuda.synchronize()
        r["dense_ms"] = e0.elapsed_time(e1) / reps
        path.attention()          # leave the sparse plan in the workspace
        torch.cuda.synchronize()
    return r


def pyramid_bytes(w, elem):
    return 2 * w.B * w.Hkv * w.N * w.d * elem * (1 + sum(2.0 ** -l for l in range(1, w.levels)))


def config_record(w, path, m, clocks, peaks_):
    """Per-preset numbers: stage times, executed TFLOP/s of the attention
    kernel as fractions of the measured burst and sustained peaks and of the
    tensor rate at the sampled clock, the pyramid's HBM fraction, the mask
    stage's roofline fraction and the dense-equivalent speedup."""
    bf16_burst, bf16_sus, hbm, src = peaks_
    elem = path.q.element_size()
    attn_tflops = m["flops"] / (m["attn_ms"] * 1e-3) / 1e12
    mhz = (clocks or {}).get("sm_mhz") or None
    pyr_gbs = pyramid_bytes(w, elem) / (m["pyr_ms"] * 1e-3) / 1e9
    rec = {"shape": "B%d Hq%d Hkv%d N%d d%d block%d L%d%s %s mask=%s" % (
               w.B, w.Hq, w.Hkv, w.N, w.d, w.block, w.levels, " causal" if w.causal else "", w.dtype, w.mask_mode),
           "ms": {"pyramid": m["pyr_ms"], "mask": m["mask_ms"], "attention": m["attn_ms"],
                  "step": m["total_ms"] / max(1, m.get("steps", 1))},
           "attn_tflops": attn_tflops, "attn_frac_of_burst": attn_tflops / bf16_burst,
           "attn_frac_of_sustained": attn_tflops / bf16_sus,
           "attn_frac_per_clock": (attn_tflops * 1e12 / (mhz * 1e6) / (TENSOR_FLOP_PER_CLK_SM * 148)) if mhz else None,
           "sm_mhz": mhz,
           "density": m["flops"] / W.dense_flops(w),
           "dense_level0_attn_ms": m["dense_ms"],
           "dense_equiv_speedup": (m["dense_ms"] / m["attn_ms"]) if m["dense_ms"] else None,
           "pyramid_gbs": pyr_gbs, "pyramid_frac_of_hbm": pyr_gbs / hbm,
           "plan_padding_frac": 1 - m["n_rows"] / max(1, 128 * m["n_tiles"])}
    if w.causal:
        fa = m["flops"] - diagonal_excess_flops(path.mask, w.N, w.block, w.d)
        rec["attn_tflops_fa_causal"] = fa / (m["attn_ms"] * 1e-3) / 1e12
        rec["fa_causal_convention"] = "only the key <= query pairs of the diagonal blocks count"
    mr = mask_roofline(w, m["mask_ms"], hbm, clocks, elem)
    if mr is not None:
        rec["mask_frac"] = mr["frac"]
        rec["mask_bound"] = "%s (%s)" % (mr["bound"], mr.get("unit_kind", mr["unit"]))
    return rec


def run_psa(args, rank, world, local_rank):
    import video_transformers_b200 as P
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workload(args)
    log(args, "generating %s inputs" % w.name)
    split = args.split == "heads" and world > 1
    q, k, v, gen = W.make_qkv(w, device=dev, seed=w.seed if split else w.seed + rank)
    if split:
        # one problem, its heads split over the ranks (every rank draws the
        # same inputs and keeps its own heads)
        hq0, hq1, hkv0, hkv1 = head_partition(w.Hq, w.Hkv, rank, world)
        q, k, v = q[:, hq0:hq1].contiguous(), k[:, hkv0:hkv1].contiguous(), v[:, hkv0:hkv1].contiguous()
        w = w.replace(name="%s[heads %d-%d of %d]" % (w.name, hq0, hq1 - 1, W.PRESETS[w.name].Hq if w.name in W.PRESETS else w.Hq),
                      Hq=hq1 - hq0, Hkv=hkv1 - hkv0)
    torch.cuda.synchronize()
    log(args, "inputs ready")
    path = Path(w, q, k, v)
    if w.mask_mode == "given":
        path.given_mask = W.make_given_mask(w, gen, device=dev)
    stream = torch.cuda.current_stream()

    if args.verbose:
        for i in range(args.warmup):
            for name, fn in (("pyramid", path.pyramid), ("mask", path.make_mask), ("attention", path.attention)):
                t = time.time()
                fn()
                torch.cuda.synchronize()
                sm = P.psa_get_device_status(path.mws)
                msg = P.psa_last_error() if sm else ""
                sa = P.psa_get_device_status(path.aws)
                msg += P.psa_last_error() if sa else ""
                log(args, "warm-up %d %s %.3f s status %d/%d %s" % (i, name, time.time() - t, sm, sa, msg))
    with ClockSampler(local_rank) as clk:
        m = measure(path, w, args, args.steps, 0 if args.verbose else args.warmup, stream, world, dev,
                    dense=not args.no_dense)
    flops = m["flops"]
    dense = W.dense_flops(w)
    n_tiles, n_rows = m["n_tiles"], m["n_rows"]
    pyr_ms, mask_ms, attn_ms, dense_ms = m["pyr_ms"], m["mask_ms"], m["attn_ms"], m["dense_ms"]
    ms_per_step = m["total_ms"] / args.steps
    if split:
        # strong scaling: the ranks share one problem; sum their work
        tot = torch.tensor([flops], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(tot)
        value = float(tot.item()) / (ms_per_step * 1e-3) / 1e12
    else:
        value = aggregate_tflops(flops, world, ms_per_step)
    gather_ms = None
    if split and not args.no_gather:
        # the full output on every rank, timed apart from the step
        torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        full = gather_heads(path.out, world)
        e1.record(stream)
        torch.cuda.synchronize()
        gather_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        del full

    # end to end through the public API with host buffers
    e2e = run_e2e(path, w, flops, args, stream) if not args.no_e2e else None

    pk = peaks()
    bf16_burst, bf16_sus, hbm, src = pk
    clocks = clk.summary()
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    pyr_bytes = pyramid_bytes(w, q.element_size())
    hist = torch.bincount(path.mask.flatten().long(), minlength=256).cpu()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp32 in, bf16 MMA",
        "data": "synthetic (smooth Gaussian field + noise, seeded)" if w.recipe == "field" else "synthetic iid N(0,1)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "block": w.block,
                   "levels": w.levels, "causal": w.causal, "mask": w.mask_mode, "policy": w.policy, "thresholds": list(w.thresholds),
                   "l2": "inputs (%.2f GB) larger than L2; no flush" % ((q.numel() + 2 * k.numel()) * q.element_size() / 1e9),
                   "step": "psa_build_pyramid + psa_make_mask + psa_attention_fwd",
                   "parallelism": ("heads split over %d GPUs (KV heads in equal runs, no data-path collective; "
                                   "all-gather of O timed apart)" % world) if split else
                                  ("replicas, one workload instance per GPU" if world > 1 else "single GPU")},
        "stages_ms": {"pyramid": pyr_ms, "mask": mask_ms, "attention": attn_ms},
        "attn_fwd_ms": attn_ms, "attn_fwd_tflops": attn_tflops,
        "executed_tflop_per_step": flops / 1e12, "dense_tflop": dense / 1e12,
        "density": flops / dense, "dense_level0_attn_ms": dense_ms,
        "dense_equiv_speedup": (dense_ms / attn_ms) if dense_ms else None,
        "level_histogram": {"l0": int(hist[0]), "l1": int(hist[1]), "l2": int(hist[2]), "l3": int(hist[3]),
                            "skip": int(hist[255])},
        "plan": {"kv_tiles": n_tiles, "real_kv_rows": n_rows, "padding_frac": 1 - n_rows / max(1, 128 * n_tiles)},
        "roofline": {"bound": "tensor", "kernel": "attn_kernel (psa_attention_fwd incl. its 3 planner kernels)",
                     "achieved": attn_tflops, "peak": bf16_sus, "unit": "TFLOP/s", "frac": attn_tflops / bf16_sus,
                     "peak_kind": "sustained bf16 (%s)" % src, "frac_of_burst": attn_tflops / bf16_burst,
                     "traffic": attn_traffic(w)},
        "pyramid_roofline": {"bound": "hbm", "achieved": pyr_bytes / (pyr_ms * 1e-3) / 1e9, "peak": hbm,
                             "unit": "GB/s", "frac": pyr_bytes / (pyr_ms * 1e-3) / 1e9 / hbm},
        "e2e": e2e,
        "gather_out_ms": gather_ms,
        "gpu_launches": launches_per_step(w) * args.steps,
        "clocks": clocks,
    }
    mr = mask_roofline(w, mask_ms, hbm, clocks, q.element_size())
    if mr is not None:
        line["mask_roofline"] = mr
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"], line["parity"] = cpu_baseline(w, q, k, v, path, args)
    if not args.no_fp8:
        line["fp8"] = measure_fp8(path, w, stream, flops, pk)
    if not args.no_backward:
        line["backward"] = measure_backward(path, w, stream, flops, pk)
    if rank == 0 and world == 1 and not args.no_configs:
        m["steps"] = args.steps
        line["configs"] = run_configs(args, w, path, m, clocks, pk, dev, stream)
    return line


def measure_backward(path, w, stream, flops_fwd, peaks_, reps=3):
    """psa_attention_bwd at the same workload and mask: the forward's output
    and lse, a random upstream gradient, then `reps` timed calls.  Its
    throughput counts 2.5x the forward's executed FLOPs (the five GEMMs of
    the forward's shape in the gradient: S, dP, dV, dK and dQ), the usual
    convention; the kernels execute more (S and dP are recomputed by the
    dQ and the dK/dV kernels, and the dK/dV tiles are level-homogeneous
    128-row tiles whose rows a query tile may not use)."""
    P = path.P
    if w.dtype != "bf16":
        return None
    dev = path.q.device
    lse = torch.empty(path.q.shape[:3], dtype=torch.float32, device=dev)
    P.psa_attention_fwd(path.shape, path.q, path.k, path.v, path.kp, path.vp, path.mask, w.sm_scale, path.out, lse,
                        path.aws)
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    dout = torch.randn(path.q.shape, generator=g, device=dev, dtype=torch.float32).to(path.q.dtype)
    dq, dk, dv = torch.empty_like(path.q), torch.empty_like(path.k), torch.empty_like(path.v)
    ws = P.workspace(P.psa_attention_bwd_workspace_bytes(path.shape), dev)

    def call():
        P.psa_attention_bwd(path.shape, path.q, path.k, path.v, path.kp, path.vp, path.mask, w.sm_scale, path.out,
                            lse, dout, dq, dk, dv, ws)
    call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    st = P.psa_get_device_status(ws)
    if st != P.PSA_OK:
        raise RuntimeError("device status %d after the backward: %s" % (st, P.psa_last_error()))
    ms = e0.elapsed_time(e1) / reps
    bf16_burst, bf16_sus = peaks_[0], peaks_[1]
    tf = 2.5 * flops_fwd / (ms * 1e-3) / 1e12
    del dq, dk, dv, ws, dout, lse
    torch.cuda.empty_cache()
    return {"entry_point": "psa_attention_bwd", "ms": ms, "reps": reps, "tflops": tf,
            "flop_convention": "2.5 x the forward's executed FLOPs", "frac_of_sustained": tf / bf16_sus,
            "frac_of_burst": tf / bf16_burst,
            "kernels": "plan (3) + prep + dq_kernel + tplan (3) + dkv_kernel + pool_bwd (2) = 11 launches"}


def measure_fp8(path, w, stream, flops_fwd, peaks_, reps=5):
    """psa_attention_fwd_fp8 (e4m3 Q and K, reading R13) and
    psa_attention_fwd_fp8_pv (e4m3 probabilities and values as well,
    reading R14) at the same workload and mask, quantization included, and
    how far each output moves from the bf16 path's."""
    P = path.P
    if w.dtype != "bf16" or w.d != 128:
        return None
    ws = P.workspace(P.psa_attention_fp8_workspace_bytes(path.shape), path.q.device)
    out8 = torch.empty_like(path.out)
    path.attention()
    torch.cuda.synchronize()
    ref = path.out.float()

    def timed(fn):
        def call():
            fn(path.shape, path.q, path.k, path.v, path.kp, path.vp, path.mask, w.sm_scale, out8, None, ws)
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(path.q.device.index or 0) as cs:
            e0.record(stream)
            for _ in range(reps):
                call()
            e1.record(stream)
            torch.cuda.synchronize()
        st = P.psa_get_device_status(ws)
        if st != P.PSA_OK:
            raise RuntimeError("device status %d after the FP8 path: %s" % (st, P.psa_last_error()))
        ms = e0.elapsed_time(e1) / reps
        diff = (out8.float() - ref).abs()
        tf = flops_fwd / (ms * 1e-3) / 1e12
        return {"ms": ms, "tflops": tf, "frac_of_burst_bf16": tf / peaks_[0], "clocks": cs.summary(),
                "vs_bf16_path": {"max_abs": diff.max().item(), "mean_abs": diff.mean().item()}}

    # peaks of the path's own MMA types: e4m3 at the nominal 2x of the measured
    # bf16 burst rate; with only S on e4m3, half the FLOPs at each rate
    fp8_peak = 2.0 * peaks_[0]
    mixed_peak = 1.0 / (0.5 / fp8_peak + 0.5 / peaks_[0])
    r = {"entry_point": "psa_attention_fwd_fp8", "reps": reps,
         "includes": "e4m3 quantization of Q and every K level, plan, attention"}
    r.update(timed(P.psa_attention_fwd_fp8))
    r["peak_own_dtype"] = {"tflops": mixed_peak, "kind": "S on e4m3 (2x the measured bf16 burst, nominal ratio), "
                           "P.V on bf16: half the FLOPs at each rate", "frac": r["tflops"] / mixed_peak}
    pv = {"entry_point": "psa_attention_fwd_fp8_pv",
          "includes": "e4m3 quantization of Q and of every K and V level, plan, attention with e4m3 P"}
    pv.update(timed(P.psa_attention_fwd_fp8_pv))
    pv["peak_own_dtype"] = {"tflops": fp8_peak, "kind": "e4m3: 2x the measured bf16 burst (nominal ratio)",
                            "frac": pv["tflops"] / fp8_peak}
    r["pv"] = pv
    del ws, out8
    torch.cuda.empty_cache()
    return r


def launches_per_step(w):
    """Kernels of ours per step: pyramid (+ blockcos), the mask stage's
    kernels, the 3 planner kernels and the attention kernel."""
    return (KERNELS_PER_STEP["pyramid"] + (1 if w.cos_min > -2 else 0) + MASK_KERNELS.get(w.mask_mode, 2)
            + KERNELS_PER_STEP["plan"] + KERNELS_PER_STEP["attention"])


def run_configs(args, w_main, path_main, m_main, clocks_main, pk, dev, stream):
    """Every preset measured the same way (the main one's numbers reused),
    each with its own parity against the oracle on a few sampled query
    blocks.  The other presets are small (about 10 ms per step)."""
    out = {}
    for name in W.ORDER:
        if name == w_main.name:
            rec = config_record(w_main, path_main, m_main, clocks_main, pk)
            out[name] = rec
            continue
        w = W.PRESETS[name]
        q, k, v, gen = W.make_qkv(w, device=dev)
        path = Path(w, q, k, v)
        if w.mask_mode == "given":
            path.given_mask = W.make_given_mask(w, gen, device=dev)
        with ClockSampler(dev.index or 0) as clk:
            m = measure(path, w, args, args.config_steps, 3, stream, dense=True)
            # keep the sampler on a little longer so short runs still get samples
            time.sleep(0.5)
        m["steps"] = args.config_steps
        rec = config_record(w, path, m, clk.summary(), pk)
        _, _, desc, par = oracle_sample(w, q, k, v, args.config_parity_blocks, seed=3, mask_dev=path.mask,
                                        gpu=path)
        rec["parity"] = dict(par, sample=desc)
        out[name] = rec
        del path, q, k, v
        torch.cuda.empty_cache()
    return out


def run_e2e(path, w, flops, args, stream):
    """The step through the public API with host buffers, as a caller that
    streams steps would run it: every step copies its Q, K, V from pinned
    host memory and reads its output and mask back to pinned host memory;
    the copies of step i + 1 and the read-back of step i overlap the compute
    of the neighbouring steps (one copy stream, one compute stream, two sets
    of device buffers used in turn).  Timed from the first copy to the last
    read-back."""
    if w.mask_mode == "given":
        return None
    dev = path.q.device
    hq = torch.empty(path.q.shape, dtype=path.q.dtype, pin_memory=True).copy_(path.q)
    hk = torch.empty(path.k.shape, dtype=path.k.dtype, pin_memory=True).copy_(path.k)
    hv = torch.empty(path.v.shape, dtype=path.v.dtype, pin_memory=True).copy_(path.v)
    ho = [torch.empty(path.out.shape, dtype=path.out.dtype, pin_memory=True) for _ in range(2)]
    hm = [torch.empty(path.mask.shape, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    paths = [path, Path(w, torch.empty_like(path.q), torch.empty_like(path.k), torch.empty_like(path.v))]
    cs, xs = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    for p in paths:
        p.stream = xs
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    steps = max(3, min(args.steps, 6))

    def run(n):
        with torch.cuda.stream(cs):
            for t, h in ((paths[0].q, hq), (paths[0].k, hk), (paths[0].v, hv)):
                t.copy_(h, non_blocking=True)
            ev_in[0].record(cs)
        for i in range(n):
            s, o = i % 2, (i + 1) % 2
            p = paths[s]
            xs.wait_event(ev_in[s])
            if i >= 2:
                xs.wait_event(ev_out[s])          # step i - 2's read-back of this set is done
            p.step()
            ev_done[s].record(xs)
            with torch.cuda.stream(cs):
                if i + 1 < n:
                    if i >= 1:
                        cs.wait_event(ev_done[o])     # step i - 1 no longer reads this set
                    for t, h in ((paths[o].q, hq), (paths[o].k, hk), (paths[o].v, hv)):
                        t.copy_(h, non_blocking=True)
                    ev_in[o].record(cs)
                cs.wait_event(ev_done[s])
                ho[s].copy_(p.out, non_blocking=True)
                hm[s].copy_(p.mask, non_blocking=True)
                ev_out[s].record(cs)

    run(2)                                          # warm-up of the second buffer set
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    run(steps)
    e1.record(cs)
    torch.cuda.synchronize()
    for p in paths:
        p.stream = None
    ms = e0.elapsed_time(e1) / steps
    del paths[1]
    torch.cuda.empty_cache()
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel()) * hq.element_size(),
            "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size() + hm[0].numel(),
            "pipelining": "copies of step i+1 and read-back of step i overlap compute (copy stream, "
                          "two device buffer sets)"}


# ----------------------------------------------------------------------------- oracle legs

def oracle_sample(w, q, k, v, n_blocks, seed=0, mask_dev=None, gpu=None):
    """The oracle on a bounded sample: one (b, h), ``n_blocks`` query blocks
    (the last, ragged one always among them).  Runs the pyramid of that
    head, the mask rows of the sample, and the attention of those rows;
    only that is timed.  Returns (seconds, executed flops, description,
    parity), where parity (when ``gpu`` holds the device path that ran the
    same workload) compares the oracle's mask rows and attention rows with
    the GPU's: mask entries that differ outside the ambiguity band, pairs in
    the band, and the max / mean abs error of the output rows."""
    import oracle.psa_oracle as O
    rng = np.random.default_rng(seed)
    b, h = 0, int(rng.integers(w.Hq))
    hk = h // (w.Hq // w.Hkv)
    n = min(n_blocks, w.nqb)
    Is = sorted(set(rng.choice(w.nqb, size=n, replace=False).tolist()) | {w.nqb - 1})
    qh = q[b:b + 1, h:h + 1].cpu()
    kh = k[b:b + 1, hk:hk + 1].cpu()
    vh = v[b:b + 1, hk:hk + 1].cpu()
    t0 = time.perf_counter()
    kl, vl = O.build_pyramid(kh, vh, w.levels)
    rows = [(0, 0, I) for I in Is]
    mass = cos = None
    if w.mask_mode == "given":
        mask = mask_dev[b:b + 1, h:h + 1].cpu().numpy()
    else:
        if w.mask_mode == "sample":
            mass = O.sampling_mass(qh, kh, w.block, w.sm_scale, w.causal, rows=rows)
        elif w.mask_mode == "meankey":
            mass = O.meankey_mass(qh, kh, w.block, w.sm_scale, w.causal, rows=rows)
        else:
            mass = O.antidiag_mass(qh, kh, w.block, w.stride, w.sm_scale, w.causal, rows=rows)
        cos = O.block_cosine(kh, w.block) if w.cos_min > -2 else None
        mask = O.make_mask(mass, w.thresholds, w.levels, w.block, w.causal, w.n_dense_prefix, cos, w.cos_min,
                           1, rows=rows, policy=w.policy)
    o, _ = O.attention(qh, kl, vl, mask, w.block, w.sm_scale, w.causal, rows=rows)
    dt = time.perf_counter() - t0
    sub = np.full_like(mask, 0xFF)
    for _, _, I in rows:
        sub[0, 0, I] = mask[0, 0, I]
    fl = O.executed_flops(sub, w.N, w.block, w.d, w.causal)
    desc = "b=0 h=%d, %d query blocks %s..., pyramid of that KV head, mask rows and attention rows" % (
        h, len(Is), Is[:4])
    if gpu is None:
        return dt, fl, desc, None
    # parity of the sampled rows (not timed)
    gmask = gpu.mask[b:b + 1, h:h + 1].cpu().numpy()
    par = {"query_blocks": len(Is), "mask_pairs": len(Is) * w.nqb}
    if mass is not None:
        th = [float(np.float32(t)) for t in w.thresholds]
        if w.policy == "quantile":
            amb = O.ambiguous_pairs_quantile(mass, th, w.levels, w.causal, 1e-6, rows=rows)
        else:
            amb = O.ambiguous_pairs(mass, th, 1e-6, rows, None if cos is None else cos, w.cos_min, 1)
        diff = np.zeros_like(amb)
        for _, _, I in rows:
            diff[0, 0, I] = gmask[0, 0, I] != mask[0, 0, I]
        par["mask_mismatch_outside_band"] = int((diff & ~amb).sum())
        par["mask_pairs_in_band"] = int(amb[0, 0, Is].sum())
        par["mask_mismatch_in_band"] = int((diff & amb).sum())
        redo = [(0, 0, I) for I in Is if diff[0, 0, I].any()]
        if redo:      # the GPU's own mask for rows whose levels legitimately differ
            o2, _ = O.attention(qh, kl, vl, gmask, w.block, w.sm_scale, w.causal, rows=redo)
            for _, _, I in redo:
                o[0, 0, I * w.block:min((I + 1) * w.block, w.N)] = o2[0, 0, I * w.block:min((I + 1) * w.block, w.N)]
    else:
        par["mask_mismatch_outside_band"] = 0
        par["mask_pairs_in_band"] = 0
    g = gpu.out[b:b + 1, h:h + 1].float().cpu().numpy().astype(np.float64)
    sel = ~np.isnan(o[..., 0])
    err = np.abs(g[sel] - o[sel])
    par["out_max_abs"] = float(err.max())
    par["out_mean_abs"] = float(err.mean())
    par["tolerance"] = {"max_abs": 2e-2, "mean_abs": 2e-3}
    par["ok"] = bool(par["mask_mismatch_outside_band"] == 0 and par["out_max_abs"] <= 2e-2
                     and par["out_mean_abs"] <= 2e-3)
    return dt, fl, desc, par


def cpu_baseline(w, q, k, v, path, args):
    dt, fl, desc, par = oracle_sample(w, q, k, v, args.cpu_blocks, mask_dev=path.mask, gpu=path)
    return ({"value": fl / dt / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
             "sample": desc, "seconds": dt}, dict(par, against="the oracle rows of cpu_baseline"))


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count()


REF_BLOCKS_TOTAL = 640


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = workload(args)
    q, k, v, gen = W.make_qkv(w, device="cuda" if torch.cuda.is_available() else "cpu")
    mask = W.make_given_mask(w, gen, device=q.device) if w.mask_mode == "given" else None
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, 1, seed=99, mask_dev=mask)[:3]
    # the whole timed run samples about REF_BLOCKS_TOTAL query blocks (about a
    # minute of host time at Wan2.1-14B size), spread over the steps
    per_step = max(1, min(args.cpu_blocks, REF_BLOCKS_TOTAL // max(1, args.steps)))
    secs, fl, desc = 0.0, 0.0, None
    for i in range(args.steps):
        dt, f, desc, _ = oracle_sample(w, q, k, v, per_step, seed=i, mask_dev=mask)
        secs += dt
        fl += f
    value = fl / secs / 1e12
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic, seeded",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                       "block": w.block, "levels": w.levels, "causal": w.causal, "mask": w.mask_mode},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": cpu_threads(),
                             "sample": "per step: " + desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def workload(args) -> W.Workload:
    """The chosen preset; --heads shrinks it (same shape per head) for
    profiling captures that must stay a few GB on the device."""
    w = W.PRESETS[args.config]
    mask_mode, policy = getattr(args, "mask_mode", "preset"), getattr(args, "policy", "mass")
    if mask_mode != "preset" or policy != "mass":
        mode = w.mask_mode if mask_mode == "preset" else mask_mode
        w = w.replace(name="%s[mask=%s,%s]" % (w.name, mode, policy), mask_mode=mode, policy=policy)
    if args.heads:
        hq = args.heads
        hkv = max(1, hq * w.Hkv // w.Hq)
        w = w.replace(name="%s[Hq=%d]" % (w.name, hq), Hq=hq, Hkv=hkv)
    return w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="wan14b", choices=W.ORDER)
    ap.add_argument("--impl", default="psa", choices=["psa", "reference"])
    ap.add_argument("--cpu-blocks", type=int, default=160, help="query blocks in the oracle sample (about 15 s of host time at Wan2.1-14B size)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-preset records of the default line")
    ap.add_argument("--no-backward", action="store_true", help="skip the timing of psa_attention_bwd")
    ap.add_argument("--no-fp8", action="store_true", help="skip the timing of psa_attention_fwd_fp8")
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: one workload instance per GPU (weak scaling) or one problem's heads split (strong)")
    ap.add_argument("--no-gather", action="store_true", help="with --split heads: skip the all-gather of O")
    ap.add_argument("--config-steps", type=int, default=10, help="timed steps per preset in the configs record")
    ap.add_argument("--config-parity-blocks", type=int, default=8,
                    help="query blocks of one head per preset checked against the oracle")
    ap.add_argument("--verbose", action="store_true", help="progress and per-stage warm-up times on stderr")
    ap.add_argument("--heads", type=int, default=0, help="override the query head count (profiling captures)")
    ap.add_argument("--mask-mode", default="preset", choices=["preset", "sample", "antidiag", "meankey"],
                    help="block scorer of the mask stage (default: the preset's)")
    ap.add_argument("--policy", default="mass", choices=["mass", "quantile"], help="level policy of the mask stage")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_psa(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
