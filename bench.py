#!/usr/bin/env python3
"""Benchmark of the relative-position-bias attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the workload's hot path over one batch of synthetic input:
for the default workload (local-layer prefill: B=2, T=8192, 32 query / 4 key-value
heads, d=128, window 512, R=512) that is one relbias_attn_fwd call writing O and
LSE.  Inputs are resident in HBM when the timed region starts; steps rotate over
several independently drawn input sets so that no step finds the previous step's
data in the 126 MB L2.  The timed region is K back-to-back steps bracketed by a
barrier and a device synchronisation on both sides and timed with CUDA events on
the launching stream; with N GPUs every rank runs its own copy of the workload
(independent units, no data-path collective: weak scaling) and the time is the max
over ranks.  Rank 0 prints one JSON line.

The default run also times every other workload (global-layer prefill at 32k and
131k tokens, decode against a 1M-token cache in its contiguous, paged and
shared-bank forms, and the local-layer backward pass), each in its own timed
region with the same rules, and reports them in the same line under "per_config".

--impl reference times the fp64 CPU oracle instead (the only other code path for
this method) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "local_prefill_bf16"
METRIC = "masked TFLOP/s & frac of bf16 tensor peak (prefill); decode HBM GB/s vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default: ~2 s of work)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token / cache length (small profiling captures only)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only --workload (the default run also times every other workload)")
    args = ap.parse_args(argv)
    args.per_config = (not args.no_per_config and args.workload == DEFAULT_WORKLOAD and args.tokens is None
                       and args.impl == "ours")
    return args


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest() -> str:
    """sha256 over the CUDA sources: ties an ncu capture to the kernels it measured."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_learned_relative_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profile_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    if that summary was taken on the current sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_%s.md" % workload)
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"source_sha256:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != source_digest():
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """Polls the SM clock and clock-event reasons through NVML while running."""

    REASONS = [("gpu_idle", 0x1), ("applications_clocks_setting", 0x2), ("sw_power_cap", 0x4),
               ("hw_slowdown", 0x8), ("sync_boost", 0x10), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80)]

    def __init__(self, torch_device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable: " + getattr(self, "error", "")]}
        names = [n for n, bit in self.REASONS if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_workload(wl, rank: int, world: int):
    """This rank's shard of an N-rank run: a global batch of world x B sequences in
    which rank r owns sequences [r*B, (r+1)*B), drawn from their own seed.  The
    shards are independent (no data-path collective); per-GPU work is fixed as the
    rank count grows (weak scaling)."""
    from dataclasses import replace
    return replace(wl, seed=wl.seed + 7919 * rank), (rank * wl.B, (rank + 1) * wl.B)


def max_over_ranks(value: float, device, world: int) -> float:
    """The largest `value` over all ranks (time of the slowest rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- our arm

def input_plan(wl):
    """Per-step input footprint, the number of independently drawn input sets the timed
    steps rotate over (enough to exceed 3x the 126 MB L2, or one set when a single step
    already does), and the note the JSON line carries about it."""
    esz = 2 if wl.dtype == "bf16" else 4
    if wl.decode:
        step_bytes = wl.kv_bytes()
    else:
        step_bytes = (2 * wl.B * wl.T * wl.Hq * wl.d + 2 * wl.B * wl.T * wl.Hkv * wl.d) * esz
        if wl.backward:   # o and dout in, fp32 gradients out
            step_bytes += 2 * wl.B * wl.T * wl.Hq * wl.d * esz + 4 * wl.B * wl.T * (wl.Hq + 2 * wl.Hkv) * wl.d
    l2 = 126 * 2 ** 20
    nsets = 1 if step_bytes > 3 * l2 else int(math.ceil(3 * l2 / step_bytes)) + 1
    note = ("%d rotating input sets (%.0f MB each) > 3x L2" % (nsets, step_bytes / 1e6)) if nsets > 1 \
        else "per-step input %.0f MB > L2" % (step_bytes / 1e6)
    return step_bytes, nsets, note


def launches_per_step(wl) -> int:
    """Kernels of this library one step launches."""
    if wl.decode:
        return 3 if wl.bank_C > 0 else 2       # (bank curves), split-KV, combine
    if wl.backward:                            # D_i, dq, dk/dv (+ bank curves, drs, dproj)
        return 6 if wl.bank_C > 0 else 3
    if wl.bank_C > 0:
        return 2                               # bank curves, prefill
    return 1                                   # the one prefill kernel


def workload_config(wl, world, l2_note):
    return {"workload": wl.name, "B": wl.B, "T": wl.T, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d,
            "window": wl.window, "R": wl.R, "global_batch": wl.B * world,
            **({"page_size": wl.page_size, "pages": "shuffled pool"} if wl.page_size > 0 else {}),
            **({"bias": "shared bank, C=%d functions" % wl.bank_C} if wl.bank_C > 0 else {}),
            **({"pass": "backward (dq, dk, dv, %s)" % ("drs, dproj" if wl.bank_C > 0 else "dr, dw")}
               if wl.backward else {}),
            "parallelism": "dp%d (batch shards, no collective)" % world,
            "l2": l2_note}


def make_sets(wl, nsets, device, shared=None):
    """`nsets` independently drawn input sets.  Decode workloads that draw the same
    cache (same seed and shape) take it from `shared` instead of drawing it again."""
    import torch
    from attention_learned_relative_b200 import workloads
    from dataclasses import replace
    sets = []
    for s in range(nsets):
        wl_s = replace(wl, seed=wl.seed + 1000 * s)
        kv = None
        key = (wl_s.seed, wl.B, wl.T, wl.Hkv, wl.d, wl.dtype, wl.qk_std)
        if wl.decode and shared is not None:
            kv = shared.get(key)
        x = workloads.make_inputs(wl_s, device=device, kv=kv)
        if wl.decode and shared is not None:
            shared[key] = (x["k"], x["v"])
        if wl.decode:
            x["o"] = torch.empty_like(x["q"])
            x["lse"] = torch.empty(wl.B, wl.Hq, dtype=torch.float32, device=device)
        elif wl.backward:
            # The forward's O and LSE are inputs of the backward: computed once, untimed.
            from attention_learned_relative_b200 import ops
            x["lse"] = torch.empty(wl.B, wl.Hq, wl.T, dtype=torch.float32, device=device)
            f32 = dict(dtype=torch.float32, device=device)
            x["g"] = {"dq": torch.empty(x["q"].shape, **f32), "dk": torch.empty(x["k"].shape, **f32),
                      "dv": torch.empty(x["v"].shape, **f32)}
            if wl.bank_C > 0:
                x["o"] = ops.attn_fwd_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], wl.window, wl.R, wl.scale,
                                           lse=x["lse"])
                x["g"].update(drs=torch.empty(x["rs"].shape, **f32), dproj=torch.empty(x["proj"].shape, **f32))
            else:
                x["o"] = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], wl.window, wl.R, wl.scale,
                                      lse=x["lse"])
                x["g"].update(dr=torch.empty(x["r"].shape, **f32), dw=torch.empty(wl.Hq, wl.R, **f32))
        else:
            x["o"] = torch.empty_like(x["q"])
            x["lse"] = torch.empty(wl.B, wl.Hq, wl.T, dtype=torch.float32, device=device)
        sets.append(x)
    return sets


def step_fn(wl, ops, workspace):
    if wl.decode and wl.page_size > 0:
        def step(x, stream):
            ops.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["table"], x["lens"], x["r"], x["w"],
                                  wl.window, wl.R, wl.T, wl.scale, out=x["o"], lse=x["lse"], workspace=workspace,
                                  stream=stream)
    elif wl.decode and wl.bank_C > 0:
        def step(x, stream):
            ops.attn_decode_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], wl.window, wl.R, wl.scale, out=x["o"],
                                 lse=x["lse"], workspace=workspace, stream=stream)
    elif wl.decode:
        def step(x, stream):
            ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], wl.window, wl.R, wl.scale, out=x["o"],
                            lse=x["lse"], workspace=workspace, stream=stream)
    elif wl.backward and wl.bank_C > 0:
        def step(x, stream):
            ops.attn_bwd_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], x["o"], x["lse"], x["dout"], wl.window,
                              wl.R, wl.scale, stream=stream, workspace=workspace, grads=x["g"])
    elif wl.bank_C > 0:
        def step(x, stream):
            ops.attn_fwd_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], wl.window, wl.R, wl.scale, out=x["o"],
                              lse=x["lse"], stream=stream, workspace=workspace)
    elif wl.backward:
        def step(x, stream):
            ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], x["o"], x["lse"], x["dout"], wl.window, wl.R,
                         wl.scale, stream=stream, workspace=workspace, grads=x["g"])
    else:
        def step(x, stream):
            ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], wl.window, wl.R, wl.scale, out=x["o"],
                         lse=x["lse"], stream=stream)
    return step


def step_outputs(wl, x):
    """The device tensors a step produces (read back to the host in the e2e measurement)."""
    if wl.backward:
        return [x["g"][n] for n in ("dq", "dk", "dv") + (("drs", "dproj") if wl.bank_C > 0 else ("dr", "dw"))]
    return [x["o"]]


def cpu_baseline(wl, x, budget_s):
    """The fp64 oracle on a bounded random sample of the workload's rows (timed on
    this host's cores).  Returns (rate, cores, description, seconds); the rate is in
    masked TFLOP/s for prefill and in GB/s of key/value cache consumed for decode."""
    import numpy as np
    import torch
    from oracle import oracle as O
    from attention_learned_relative_b200.workloads import logical_cache

    g = torch.Generator().manual_seed(12345)
    if wl.decode:
        # Rows of decode span the whole cache: sample (sequence, key/value head)
        # groups and copy only that group's cache slice to the host.
        G = wl.group
        t_all, nbytes, groups = 0.0, 0.0, 0
        while t_all < budget_s and groups < 64:
            b = int(torch.randint(0, wl.B, (1,), generator=g))
            kv = int(torch.randint(0, wl.Hkv, (1,), generator=g))
            heads = list(range(kv * G, (kv + 1) * G))
            k_sl, v_sl = logical_cache(x, b, kv)
            k_sl, v_sl = k_sl[None].cpu(), v_sl[None].cpu()
            q = x["q"][b, heads].float().cpu()
            if wl.bank_C > 0:
                r = x["rs"][b, heads].cpu()              # [G, C]
                proj = x["proj"].cpu()                   # [1, C, R], shared by the heads
            else:
                r = x["r"][b, heads].cpu().reshape(G, 1)
                proj = x["w"][heads].cpu().reshape(G, 1, wl.R)
            req = np.array([(0, hl, wl.T - 1) for hl in range(G)], dtype=np.int64)
            t0 = time.perf_counter()
            O.attn_rows(q, r, proj, k_sl, v_sl, req, G, wl.window, wl.R, wl.scale)
            t_all += time.perf_counter() - t0
            nbytes += 2 * wl.attended_pairs() * wl.d * (2 if wl.dtype == "bf16" else 4)
            groups += 1
        return nbytes / t_all / 1e9, O.num_threads(), \
            "%d (sequence, kv-head) groups of %s, all %d query heads each over the full cache (%.1f s)" % (
                groups, wl.name, G, t_all), t_all

    if wl.backward:
        # The oracle's backward over a prefix of sequence 0 (all heads): causal, so the
        # prefix is a complete sub-problem.  Its length is sized to the time budget.
        def run(n):
            bias = ("rs", "proj") if wl.bank_C > 0 else ("r", "w")
            args = [x[t][:1, :n].cpu() for t in ("q", "k", "v", bias[0])]
            t0 = time.perf_counter()
            O.attn_backward(args[0], args[1], args[2], args[3], x[bias[1]].cpu(), x["dout"][:1, :n].cpu(), wl.window,
                            wl.R, wl.scale)
            return time.perf_counter() - t0

        def pairs(n):
            W = wl.window
            return n * (n + 1) // 2 if (W <= 0 or W >= n) else W * (W + 1) // 2 + (n - W) * W

        n0 = min(256, wl.T)
        t_small = max(run(n0), 1e-4)
        per_pair = t_small / pairs(n0)
        n = n0
        while n < wl.T and pairs(min(wl.T, 2 * n)) * per_pair <= budget_s:
            n = min(wl.T, 2 * n)
        dt = run(n)
        fl = 10.0 * wl.d * pairs(n) * wl.Hq
        return fl / dt / 1e12, O.num_threads(), \
            "backward of the first %d tokens of sequence 0 of %s, all %d heads (%.3g masked GFLOP, %.1f s)" % (
                n, wl.name, wl.Hq, fl / 1e9, dt), dt

    k_cpu = x["k"].cpu()
    v_cpu = x["v"].cpu()
    if wl.bank_C > 0:
        proj = x["proj"].cpu()                       # [1, C, R], shared by the heads
        coef = x["rs"]                               # [B, T, Hq, C]
    else:
        proj = x["w"].cpu().reshape(wl.Hq, 1, wl.R)
        coef = x["r"][..., None]                     # [B, T, Hq, 1]

    def draw(n):
        b = torch.randint(0, wl.B, (n,), generator=g)
        h = torch.randint(0, wl.Hq, (n,), generator=g)
        i = torch.randint(0, wl.T, (n,), generator=g)
        idx = [t.to(x["q"].device) for t in (b, i, h)]
        q = x["q"][idx[0], idx[1], idx[2]].float().cpu()
        r = coef[idx[0], idx[1], idx[2]].cpu()
        rows = torch.stack([b, h, i], 1).numpy().astype(np.int64)
        return rows, q, r.reshape(n, -1)

    def flops(rows):
        i = rows[:, 2]
        n = i + 1 if wl.window <= 0 else np.minimum(i + 1, wl.window)
        return float(4 * wl.d * n.sum())

    rows, q, r = draw(8)
    O.attn_rows(q, r, proj, k_cpu, v_cpu, rows, wl.Hq, wl.window, wl.R, wl.scale)   # load, warm up
    rows, q, r = draw(256)
    t0 = time.perf_counter()
    O.attn_rows(q, r, proj, k_cpu, v_cpu, rows, wl.Hq, wl.window, wl.R, wl.scale)
    per_row = max((time.perf_counter() - t0) / len(rows), 1e-6)
    n = int(max(8, min(4000000, budget_s / per_row)))
    rows, q, r = draw(n)
    t0 = time.perf_counter()
    O.attn_rows(q, r, proj, k_cpu, v_cpu, rows, wl.Hq, wl.window, wl.R, wl.scale)
    dt = time.perf_counter() - t0
    return flops(rows) / dt / 1e12, O.num_threads(), \
        "%d random (b,h,i) rows of %s (%.3g masked GFLOP, %.1f s)" % (n, wl.name, flops(rows) / 1e9, dt), dt


# Workloads the default run measures beside the headline one, each in its own timed
# region, reported in the same JSON line under "per_config".
PER_CONFIG = ["local_prefill_bank_bf16", "global_prefill_bf16", "global_long_prefill_bf16", "global_decode_bf16",
              "global_decode_paged_bf16", "global_decode_bank_bf16", "local_backward_bf16",
              "local_backward_bank_bf16"]


def roofline_of(wl, ms_step, peaks, peaks_kind):
    """Roofline object of a workload's dominant kernel(s) at `ms_step` per step."""
    traffic = profile_traffic(wl.name)
    if wl.decode:
        per_step = wl.kv_bytes()
        achieved = per_step / (ms_step * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        return per_step, {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                          "traffic": traffic, "peak_source": peaks_kind + " hbm_gbs (copy)",
                          "kernel": ("bank_curves_kernel + " if wl.bank_C > 0 else "")
                          + "decode_splitkv_kernel + decode_combine_kernel",
                          "algorithmic_bytes_per_launch": per_step}
    per_step = wl.masked_flops()
    achieved = per_step / (ms_step * 1e-3) / 1e12
    # bf16 runs on the tcgen05 tensor cores (the backward too, for d in {64, 128});
    # fp32 on CUDA cores: 148 SMs x 128 FMA lanes x 2 flop x 1.965 GHz.
    tensor = wl.dtype == "bf16" and (not wl.backward or wl.d in (64, 128))
    peak = float(peaks["bf16_tflops"]) if tensor else 148 * 128 * 2 * 1.965e9 / 1e12
    if wl.backward:
        kernel = "bwd_dq_sm100_kernel + bwd_dkv_sm100_kernel" if tensor else "bwd_dq_kernel + bwd_dkv_kernel"
        if wl.bank_C > 0:
            kernel = "bank_rows_kernel + " + kernel + " + bank_drs_kernel + bank_dproj_kernel"
    elif wl.dtype == "bf16":
        kernel = "bank_rows_kernel + prefill_bf16_sm100_kernel" if wl.bank_C > 0 else "prefill_bf16_sm100_kernel"
    else:
        kernel = "prefill_fp32_kernel"
    return per_step, {"bound": "tensor" if tensor else "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                      "frac": achieved / peak, "traffic": traffic,
                      "peak_source": (peaks_kind + " bf16_tflops (burst)") if tensor
                      else "fp32 FMA units x max clock",
                      "frac_of_datasheet_2250": achieved / 2250.0,
                      "kernel": kernel,
                      "algorithmic_flops_per_launch": per_step}


def measure(args, wl, ctx, steps_arg, e2e_on, cpu_budget, shared=None):
    """Time one workload: W warm-up steps, then K steps between barriers and device
    synchronisations, CUDA events on the launching stream, max over ranks.  Every rank
    takes the same collective steps.  Returns the JSON object on rank 0, else None."""
    import torch
    from attention_learned_relative_b200 import ops

    rank, world, dev = ctx["rank"], ctx["world"], ctx["dev"]
    step_bytes, nsets, l2_note = input_plan(wl)
    wl_r, _ = rank_workload(wl, rank, world)
    sets = make_sets(wl_r, nsets, dev, shared)
    workspace = None
    if wl.backward and wl.bank_C > 0:
        workspace = torch.empty(max(256, ops.lib().relbias_attn_bwd_bank_workspace_size(wl.B, wl.T, wl.Hq, wl.R)),
                                dtype=torch.uint8, device=dev)
    elif wl.backward:
        workspace = torch.empty(max(16, ops.lib().relbias_attn_bwd_workspace_size(wl.B, wl.T, wl.Hq)),
                                dtype=torch.uint8, device=dev)
    elif wl.bank_C > 0 and not wl.decode:
        nbytes = ops.fwd_bank_workspace_size(wl.B, wl.T, wl.Hq, wl.R,
                                             ops.RELBIAS_BF16 if wl.dtype == "bf16" else ops.RELBIAS_FP32)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    if wl.decode:
        if wl.page_size > 0:
            nbytes = ops.decode_paged_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.window)
        elif wl.bank_C > 0:
            nbytes = ops.decode_bank_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.window, wl.R)
        else:
            nbytes = ops.decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.window)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    step = step_fn(wl_r, ops, workspace)
    stream = torch.cuda.current_stream(dev)

    # Warm-up; then size the timed region to ~2 s unless --steps is given.
    t0 = time.perf_counter()
    for i in range(max(args.warmup, 1)):
        step(sets[i % nsets], stream)
    torch.cuda.synchronize()
    warm_ms = (time.perf_counter() - t0) * 1e3 / max(args.warmup, 1)
    steps = steps_arg if steps_arg is not None else int(max(20, min(20000, 2000.0 / max(warm_ms, 1e-3))))
    # The step count is the same on every rank (rank 0's choice).
    steps = int(round(max_over_ranks(float(steps), dev, world))) if world > 1 else steps
    ops.device_status(reset=True)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(ctx["local"]) as clocks:
        ev0.record(stream)
        for i in range(steps):
            step(sets[i % nsets], stream)
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_total = ev0.elapsed_time(ev1)
    status = ops.device_status(reset=True)
    ms_total = max_over_ranks(ms_total, dev, world)
    ms_step = ms_total / steps

    # End to end through the public API: pinned host inputs -> device -> kernel -> host.
    e2e = None
    if e2e_on:
        x = sets[0]
        if wl.decode:
            names_in = ["q", "rs"] if wl.bank_C > 0 else ["q", "r"]
        elif wl.backward:
            names_in = ["q", "k", "v"] + (["rs", "proj"] if wl.bank_C > 0 else ["r", "w"]) + ["o", "lse", "dout"]
        elif wl.bank_C > 0:
            names_in = ["q", "k", "v", "rs", "proj"]
        else:
            names_in = ["q", "k", "v", "r", "w"]
        host_in = {n: x[n].cpu().pin_memory() for n in names_in}
        dev_out = step_outputs(wl, x)
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in dev_out]
        bi = sum(t.numel() * t.element_size() for t in host_in.values())
        bo = sum(t.numel() * t.element_size() for t in host_out)
        e2e_steps = max(3, min(steps, 50))

        def e2e_step():
            for n, t in host_in.items():
                x[n].copy_(t, non_blocking=True)
            step(x, stream)
            for h_, d_ in zip(host_out, dev_out):
                h_.copy_(d_, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev, world)
        e2e = {"e_ms": e_ms, "bi": bi, "bo": bo}

    result = None
    if rank == 0:
        per_step, roof = roofline_of(wl, ms_step, ctx["peaks"], ctx["peaks_kind"])
        unit = roof["unit"]
        value = per_step * world / (ms_step * 1e-3) / (1e9 if wl.decode else 1e12)
        result = {
            "metric": METRIC,
            "value": value,
            "unit": unit,
            "n_gpus": world,
            "steps": steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": wl.dtype,
            "data": "synthetic",
            "config": workload_config(wl, world, l2_note),
            "roofline": roof,
            "clocks": clocks.summary(),
            "gpu_launches": steps * launches_per_step(wl),
            "kernel_status": status,
        }
        if e2e is not None:
            e_val = per_step * world / (e2e["e_ms"] * 1e-3) / (1e9 if wl.decode else 1e12)
            result["e2e"] = {"value": e_val, "unit": unit, "h2d_bytes_per_step": e2e["bi"],
                             "d2h_bytes_per_step": e2e["bo"], "ms_per_step": e2e["e_ms"]}
        if world == 1 and cpu_budget is not None:
            v, cores, desc, _ = cpu_baseline(wl, sets[0], cpu_budget)
            result["cpu_baseline"] = {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": desc}
    del sets, workspace
    return result


def run_ours(args, wl, peaks, peaks_kind):
    import torch
    import torch.distributed as dist
    from attention_learned_relative_b200 import build
    from attention_learned_relative_b200.workloads import WORKLOADS

    rank, world, local = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
    build.build()  # no-op when the in-tree library is current
    ctx = {"rank": rank, "world": world, "local": local, "dev": dev, "peaks": peaks, "peaks_kind": peaks_kind}

    cpu_budget = None if args.no_cpu_baseline else args.cpu_seconds
    result = measure(args, wl, ctx, args.steps, not args.no_e2e, cpu_budget)
    torch.cuda.empty_cache()

    if args.per_config:
        per = {}
        shared = {}
        for name in PER_CONFIG:
            pwl = WORKLOADS[name]
            r = measure(args, pwl, ctx, args.steps, False,
                        None if cpu_budget is None else min(cpu_budget, 4.0), shared)
            if rank == 0:
                per[name] = {k: r[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config",
                                               "roofline", "clocks", "gpu_launches", "kernel_status")}
                if "cpu_baseline" in r:
                    per[name]["cpu_baseline"] = r["cpu_baseline"]
            if not pwl.decode:
                shared.clear()
            torch.cuda.empty_cache()
        shared.clear()
        if rank == 0:
            result["per_config"] = per
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, wl, steps_default=5):
    """The fp64 CPU oracle, as it stands, timed on this host's cores: each step is a
    bounded random sample of the workload's rows (inputs drawn on the GPU when one is
    present, else on the CPU)."""
    import torch
    from attention_learned_relative_b200 import workloads
    from oracle import oracle as O

    O.build()
    steps = args.steps if args.steps is not None else steps_default
    warm = max(args.warmup, 0)
    per_step_s = max(0.5, min(5.0, 150.0 / max(1, steps + warm)))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = workloads.make_inputs(wl, device=dev)
    tot_work = 0.0
    tot_s = 0.0
    desc = None
    cores = O.num_threads()
    for s in range(warm + steps):
        rate, cores, desc, dt = cpu_baseline(wl, x, per_step_s)
        if s >= warm:
            tot_work += rate * dt
            tot_s += dt
    value = tot_work / tot_s
    unit = "GB/s" if wl.decode else "TFLOP/s"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": 1, "steps": steps,
        "warmup": warm, "ms_per_step": tot_s * 1e3 / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, 1, input_plan(wl)[2]),
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    from attention_learned_relative_b200.workloads import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.tokens is not None:
        from dataclasses import replace
        wl = replace(wl, T=args.tokens)
    peaks, kind = load_peaks()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args, wl)), flush=True)
        return 0
    res = run_ours(args, wl, peaks, kind)
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
