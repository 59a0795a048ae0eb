"""GPU parity of the prefill entry point (relbias_attn_fwd) against the fp64 oracle.

Small cases are compared element by element over every output; they span several
128-row tiles, a ragged tail, single-slot (odd GQA group) and two-slot work items,
d = 64 and 128, sliding windows, R = 0 / 1 / within / beyond the window.  The full
workloads run in the same launch configuration the benchmark times and are
compared on sampled rows (tile edges, bias and window boundaries, random rows).
"""
import math

import numpy as np
import pytest
import torch

from attention_learned_relative_b200 import ops, synth
from attention_learned_relative_b200.workloads import WORKLOADS, make_inputs
from oracle import oracle as O
from parity import assert_bf16_close, assert_fp32_close, sample_rows

pytestmark = pytest.mark.gpu


def _inputs(B, T, Hq, Hkv, d, R, seed, dtype=torch.bfloat16, qk_std=1.0):
    dev = "cuda"
    return {
        "q": synth.normal((B, T, Hq, d), seed, "q", std=qk_std, dtype=dtype, device=dev),
        "k": synth.normal((B, T, Hkv, d), seed, "k", std=qk_std, dtype=dtype, device=dev),
        "v": synth.normal((B, T, Hkv, d), seed, "v", dtype=dtype, device=dev),
        "r": synth.normal((B, T, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
    }


def _run(x, window, R, scale):
    B, T, Hq, _ = x["q"].shape
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, scale, lse=lse)
    torch.cuda.synchronize()
    return o, lse


def _oracle(x, window, R, scale):
    return O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), window, R, scale)


@pytest.fixture(autouse=True)
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out"


def test_tiny_local_fp32_workload():
    wl = WORKLOADS["tiny_local_fp32"]
    x = make_inputs(wl, device="cuda")
    o, lse = _run(x, wl.window, wl.R, wl.scale)
    o_ref, lse_ref = _oracle(x, wl.window, wl.R, wl.scale)
    assert_fp32_close(o, o_ref, lse, lse_ref, wl.name)


@pytest.mark.parametrize("d", [32, 64, 128, 256])
@pytest.mark.parametrize("window,R", [(0, 50), (33, 64), (100, 10)])
def test_fp32_shapes(d, window, R):
    x = _inputs(2, 97, 4, 2, d, R, seed=11 + d, dtype=torch.float32)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(x, window, R, scale)
    o_ref, lse_ref = _oracle(x, window, R, scale)
    assert_fp32_close(o, o_ref, lse, lse_ref, "fp32 d=%d" % d)


BF16_CASES = [
    # B, T,    Hq, Hkv, d,   window, R
    (1, 300, 8, 2, 128, 0, 64),        # causal, ragged tail, two-slot items
    (2, 700, 8, 2, 128, 512, 512),     # local layer shape
    (1, 1100, 4, 1, 128, 0, 1024),     # global layer: bias over 1024, content-only beyond
    (1, 513, 2, 2, 128, 128, 100),     # GQA group 1: single-slot items
    (1, 640, 6, 2, 128, 300, 37),      # GQA group 3: single-slot items
    (1, 400, 8, 1, 64, 0, 200),        # head dim 64
    (1, 257, 4, 2, 64, 64, 64),
    (1, 1, 8, 1, 128, 0, 16),          # one token
    (1, 127, 4, 2, 128, 0, 300),
    (1, 128, 4, 2, 128, 0, 128),
    (1, 129, 4, 2, 128, 0, 129),
    (1, 333, 4, 2, 128, 0, 0),         # R = 0: no bias at all
    (1, 333, 4, 2, 128, 0, 1),         # R = 1: only the diagonal
    (1, 333, 4, 2, 128, 1, 8),         # window 1: each row sees itself
    (1, 600, 4, 4, 128, 700, 2048),    # window wider than the sequence, largest R
]


@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R", BF16_CASES)
def test_bf16_parity(B, T, Hq, Hkv, d, window, R):
    x = _inputs(B, T, Hq, Hkv, d, R, seed=T + 7 * R + window)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(x, window, R, scale)
    o_ref, lse_ref = _oracle(x, window, R, scale)
    assert_bf16_close(o, o_ref, lse, lse_ref, "bf16 %s" % ((B, T, Hq, Hkv, d, window, R),))


def test_bf16_other_scale_and_large_logits():
    """scale 1/d (the essay's alternative reading) and a steep bias that forces the
    running max to jump between tiles (rescale path)."""
    B, T, Hq, Hkv, d, R = 1, 900, 4, 2, 128, 900
    x = _inputs(B, T, Hq, Hkv, d, R, seed=5)
    x["w"] = x["w"] * 12.0
    x["w"][:, 600:] += 30.0     # keys 600+ back become much more likely once reached
    for scale in (1.0 / d, 0.3):
        o, lse = _run(x, 0, R, scale)
        o_ref, lse_ref = _oracle(x, 0, R, scale)
        assert_bf16_close(o, o_ref, lse, lse_ref, "scale %g" % scale)


@pytest.mark.parametrize("dtype,B,T,Hq,Hkv,d,window,R,n0", [
    (torch.bfloat16, 1, 700, 8, 2, 128, 0, 256, 200),      # global layer: rows past 200 keys are sharpened
    (torch.bfloat16, 1, 900, 4, 2, 128, 512, 512, 300),    # windowed: n saturates at the window
    (torch.bfloat16, 1, 400, 8, 1, 64, 0, 64, 50),
    (torch.float32, 1, 300, 4, 2, 64, 0, 64, 40),
    (torch.float32, 1, 300, 4, 2, 128, 100, 30, 20),
])
def test_context_length_temperature(dtype, B, T, Hq, Hkv, d, window, R, n0):
    """Logits of a row that sees n > n0 keys scaled by ln n / ln n0 (content and bias)."""
    x = _inputs(B, T, Hq, Hkv, d, R, seed=T + n0, dtype=dtype)
    scale = 1.0 / math.sqrt(d)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, scale, lse=lse, temp_n0=n0)
    torch.cuda.synchronize()
    o_ref, lse_ref = O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), window,
                                    R, scale, temp_n0=n0)
    check = assert_fp32_close if dtype == torch.float32 else assert_bf16_close
    check(o, o_ref, lse, lse_ref, "temperature %s" % ((dtype, B, T, Hq, Hkv, d, window, R, n0),))


def test_temperature_off_is_bitwise_identical():
    """A break point that no row's key count exceeds leaves every output bit unchanged."""
    x = _inputs(1, 500, 8, 2, 128, 128, seed=41)
    o0, l0 = _run(x, 0, 128, 0.09)
    for n0 in (1, 500, 100000):
        lse = torch.empty_like(l0)
        o1 = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], 0, 128, 0.09, lse=lse, temp_n0=n0)
        torch.cuda.synchronize()
        assert torch.equal(o0, o1) and torch.equal(l0, lse)


def test_deterministic():
    x = _inputs(1, 1000, 8, 2, 128, 512, seed=3)
    o1, l1 = _run(x, 512, 512, 0.088)
    o2, l2 = _run(x, 512, 512, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_window_locality_is_bitwise():
    """Changing keys/values older than the window leaves later rows bit-identical:
    the kernel never reads tiles outside the window for them."""
    T, W = 1500, 256
    x = _inputs(1, T, 8, 2, 128, W, seed=21)
    o1, l1 = _run(x, W, W, 0.09)
    x2 = dict(x)
    x2["k"] = x["k"].clone()
    x2["v"] = x["v"].clone()
    x2["k"][:, :400] = 3.0
    x2["v"][:, :400] = -7.0
    o2, l2 = _run(x2, W, W, 0.09)
    first_free = 400 + W - 1
    assert torch.equal(o1[:, first_free:], o2[:, first_free:])
    assert torch.equal(l1[:, :, first_free:], l2[:, :, first_free:])
    assert not torch.equal(o1[:, first_free - 1], o2[:, first_free - 1])


def test_output_buffers_fully_written():
    x = _inputs(1, 300, 4, 2, 128, 64, seed=9)
    out = torch.full_like(x["q"], float("nan"))
    lse = torch.full((1, 4, 300), float("nan"), device="cuda")
    ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], 0, 64, 0.1, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_output_alignment_paths_agree():
    """O 32-byte aligned (written with 32-byte stores) and O only 16-byte aligned (16-byte
    stores) give bit-identical results, rows of a ragged last tile included."""
    x = _inputs(2, 333, 8, 2, 128, 128, seed=31)
    o_a = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], 0, 128, 0.09)
    flat = torch.empty(x["q"].numel() + 8, dtype=x["q"].dtype, device="cuda")
    o_u = flat[8:].view(x["q"].shape)              # 16 bytes past a 256-byte aligned base
    assert o_a.data_ptr() % 32 == 0 and o_u.data_ptr() % 32 == 16
    ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], 0, 128, 0.09, out=o_u)
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_u)


def _sampled_check(wl, per_head, seed):
    x = make_inputs(wl, device="cuda")
    B, T, Hq, d = x["q"].shape
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], wl.window, wl.R, wl.scale, lse=lse)
    torch.cuda.synchronize()
    rows = sample_rows(B, T, Hq, per_head, seed, extra=(wl.R - 1, wl.R, wl.R + 1, wl.window - 1, wl.window))
    idx = torch.as_tensor(rows, device="cuda")
    q_rows = x["q"][idx[:, 0], idx[:, 2], idx[:, 1]].float().cpu()
    rs_rows = x["r"][idx[:, 0], idx[:, 2], idx[:, 1]].cpu().reshape(-1, 1)
    proj = x["w"].cpu().reshape(Hq, 1, wl.R)
    o_ref, lse_ref = O.attn_rows(q_rows, rs_rows, proj, x["k"].cpu(), x["v"].cpu(), rows, Hq, wl.window, wl.R,
                                 wl.scale)
    o_rows = o[idx[:, 0], idx[:, 2], idx[:, 1]]
    lse_rows = lse[idx[:, 0], idx[:, 1], idx[:, 2]]
    return assert_bf16_close(o_rows, o_ref, lse_rows, lse_ref, wl.name)


def test_local_prefill_workload_sampled():
    _sampled_check(WORKLOADS["local_prefill_bf16"], per_head=24, seed=1)


def test_global_prefill_workload_sampled():
    _sampled_check(WORKLOADS["global_prefill_bf16"], per_head=12, seed=2)


def test_global_long_prefill_workload_sampled():
    _sampled_check(WORKLOADS["global_long_prefill_bf16"], per_head=4, seed=3)
