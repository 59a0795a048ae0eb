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


def test_committed_ncu_summaries_carry_their_source_digest(monkeypatch):
    """Every ncu summary under profiles/ names the digest of the CUDA sources it was taken
    on, and most give DRAM bytes per launch.  The benchmark uses those bytes as the
    roofline's `traffic` only while the digest matches the sources in the tree; a stale
    summary, or one without the figure, gives null."""
    import re
    prof = os.path.join(ROOT, "profiles")
    found = 0
    for name in sorted(os.listdir(prof)):
        if not name.startswith("ncu_"):
            continue
        text = open(os.path.join(prof, name)).read()
        m = re.search(r"source_sha256:\s*([0-9a-f]{16})", text)
        assert m, name
        has_bytes = re.search(r"dram_bytes_per_launch:\s*[0-9.eE+]+", text) is not None
        workload = name[len("ncu_"):-len(".md")]
        assert workload in WORKLOADS, name
        current = m.group(1) == bench.source_digest() and has_bytes
        assert (bench.profile_traffic(workload) is not None) == current, name
        monkeypatch.setattr(bench, "source_digest", lambda: "0" * 16)
        assert bench.profile_traffic(workload) is None, name
        monkeypatch.undo()
        found += 1
    assert found >= 3


def test_default_run_times_every_workload_in_one_line():
    """The default invocation (no arguments) measures the headline workload and every
    workload in PER_CONFIG; any other --workload times only itself."""
    a = bench.parse_args([])
    assert a.per_config and a.workload == bench.DEFAULT_WORKLOAD
    assert not bench.parse_args(["--workload", "global_prefill_bf16"]).per_config
    assert not bench.parse_args(["--no-per-config"]).per_config
    assert not bench.parse_args(["--tokens", "1024"]).per_config
    assert not bench.parse_args(["--impl", "reference"]).per_config
    names = set(bench.PER_CONFIG)
    assert names <= set(WORKLOADS) and bench.DEFAULT_WORKLOAD not in names
    for want in ("global_prefill_bf16", "global_long_prefill_bf16", "global_decode_bf16",
                 "global_decode_paged_bf16", "global_decode_bank_bf16"):
        assert want in names


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_input_plan_exceeds_l2(name):
    """Steps rotate over enough input sets that their footprint exceeds 3x the L2, or one
    step alone exceeds it."""
    wl = WORKLOADS[name]
    step_bytes, nsets, note = bench.input_plan(wl)
    l2 = 126 * 2 ** 20
    assert step_bytes * nsets > 3 * l2 or (nsets == 1 and step_bytes > 3 * l2)
    cfg = bench.workload_config(wl, 1, note)
    assert cfg["workload"] == name and cfg["l2"] == note and cfg["global_batch"] == wl.B
    assert bench.launches_per_step(wl) >= 1
