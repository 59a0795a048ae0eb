"""The benchmark's CPU-baseline leg (the oracle timed on a bounded sample) on small
copies of every workload kind: prefill, decode, paged decode, shared-bank decode and
the backward pass.  No GPU: inputs are drawn on the CPU."""
import os
import sys
from dataclasses import replace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from attention_learned_relative_b200.workloads import WORKLOADS, make_inputs  # noqa: E402


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_cpu_baseline_runs_on_every_workload_kind(name):
    wl = WORKLOADS[name]
    small = replace(wl, B=min(wl.B, 2), T=min(wl.T, 512), R=min(wl.R, 256),
                    window=min(wl.window, 128) if wl.window > 0 else wl.window)
    x = make_inputs(small, device="cpu")
    rate, cores, desc, dt = bench.cpu_baseline(small, x, 0.05)
    assert rate > 0 and cores >= 1 and dt > 0
    assert small.name in desc


def test_backward_flops_are_two_and_a_half_forwards():
    fwd = WORKLOADS["local_prefill_bf16"]
    bwd = WORKLOADS["local_backward_bf16"]
    assert bwd.masked_flops() * 2 == fwd.masked_flops() * 5


@pytest.mark.parametrize("T,window", [(1, 0), (7, 0), (100, 0), (100, 1), (100, 17), (100, 100), (100, 250)])
def test_attended_pairs_match_a_brute_force_count(T, window):
    """The FLOP count the benchmark divides by: pairs (i, j) with 0 <= i - j and, for a
    window, i - j < window, counted one by one."""
    wl = replace(WORKLOADS["tiny_local_fp32"], T=T, window=window, B=3, Hq=5, d=16)
    brute = sum(1 for i in range(T) for j in range(T) if 0 <= i - j and (window <= 0 or i - j < window))
    assert wl.attended_pairs() == brute
    assert wl.masked_flops() == 4 * 16 * brute * 3 * 5


def test_decode_bytes_are_the_attended_cache_rows():
    wl = WORKLOADS["global_decode_bf16"]
    assert wl.attended_pairs() == wl.T
    assert wl.kv_bytes() == 2 * wl.B * wl.Hkv * wl.T * wl.d * 2
    win = replace(wl, window=512)
    assert win.kv_bytes() == 2 * wl.B * wl.Hkv * 512 * wl.d * 2


def test_committed_ncu_summaries_describe_the_current_kernels():
    """Every ncu summary under profiles/ names the digest of the CUDA sources it was taken
    on; it must be the digest of the sources in the tree."""
    import re
    prof = os.path.join(ROOT, "profiles")
    found = 0
    for name in sorted(os.listdir(prof)):
        if not name.startswith("ncu_"):
            continue
        m = re.search(r"source_sha256:\s*([0-9a-f]+)", open(os.path.join(prof, name)).read())
        assert m, name
        assert m.group(1) == bench.source_digest(), name
        found += 1
    assert found >= 3
