"""Failure detection on the GPU without a fault: the kernels' bounded waits.

Every wait inside the prefill and decode kernels gives up after a limit (2 s by
default), records RELBIAS_STATUS_TIMEOUT in the device status word, and the kernel
winds down: the TMA producer waits for the copies it issued, the MMA warp for its
MMAs, tensor memory is released and the kernel returns.  These tests lower the limit
through the C ABI to a nanosecond, so that ordinary waits on copies and MMAs run out,
and check that the status comes back, that the call returns, and that the next call
with the default limit is clean and correct.  Nothing here faults, traps or hangs a
GPU: the waits that run out are the kernels' own bounded waits.
"""
import math

import numpy as np

import pytest
import torch

from attention_learned_relative_b200 import ops, synth
from oracle import oracle as O
from parity import assert_bf16_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _restore_limit():
    ops.device_status(reset=True)
    yield
    ops.set_wait_limit_ns(0)
    ops.device_status(reset=True)


def _prefill_inputs(B, T, Hq, Hkv, d, R, seed):
    dev = "cuda"
    return (synth.normal((B, T, Hq, d), seed, "q", dtype=torch.bfloat16, device=dev),
            synth.normal((B, T, Hkv, d), seed, "k", dtype=torch.bfloat16, device=dev),
            synth.normal((B, T, Hkv, d), seed, "v", dtype=torch.bfloat16, device=dev),
            synth.normal((B, T, Hq), seed, "r", device=dev),
            synth.normal((Hq, R), seed, "w", std=0.5, device=dev))


@pytest.mark.parametrize("window,R", [(512, 512), (0, 1024)])
def test_prefill_wait_runs_out_then_next_call_is_clean(window, R):
    B, T, Hq, Hkv, d = 1, 4096, 32, 4, 128
    q, k, v, r, w = _prefill_inputs(B, T, Hq, Hkv, d, R, seed=31)
    ops.set_wait_limit_ns(1)
    for _ in range(3):
        ops.attn_fwd(q, k, v, r, w, window, R, 1.0 / math.sqrt(d))
    status = ops.device_status(reset=True)          # synchronises: the kernels returned
    assert status & ops.RELBIAS_STATUS_TIMEOUT, "no wait ran out under a 1 ns limit"

    ops.set_wait_limit_ns(0)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(q, k, v, r, w, window, R, 1.0 / math.sqrt(d), lse=lse)
    assert ops.device_status(reset=True) == 0
    rows = [(0, h, i) for h in (0, 17, 31) for i in (0, 127, 128, 1000, 4095)]
    req = np.array(rows, dtype=np.int64)
    o_ref, lse_ref = O.attn_rows(q[0, :, :].float().cpu()[req[:, 2], req[:, 1]], r.cpu()[0][req[:, 2], req[:, 1]]
                                 .reshape(-1, 1), w.cpu().reshape(Hq, 1, R), k.cpu(), v.cpu(), req, Hq, window, R,
                                 1.0 / math.sqrt(d))
    got = o[0].float().cpu()[req[:, 2], req[:, 1]]
    got_lse = lse[0].cpu()[req[:, 1], req[:, 2]]
    assert_bf16_close(got, o_ref, got_lse, lse_ref, "prefill after a timed-out call")


def test_decode_wait_runs_out_then_next_call_is_clean():
    B, N, Hq, Hkv, d, R = 4, 200000, 32, 4, 128, 1024
    dev = "cuda"
    q = synth.normal((B, Hq, d), 9, "q", dtype=torch.bfloat16, device=dev)
    k = synth.normal((B, N, Hkv, d), 9, "k", dtype=torch.bfloat16, device=dev)
    v = synth.normal((B, N, Hkv, d), 9, "v", dtype=torch.bfloat16, device=dev)
    r = synth.normal((B, Hq), 9, "r", device=dev)
    w = synth.normal((Hq, R), 9, "w", std=0.5, device=dev)
    ops.set_wait_limit_ns(1)
    for _ in range(3):
        ops.attn_decode(q, k, v, r, w, 0, R, 0.1)
    assert ops.device_status(reset=True) & ops.RELBIAS_STATUS_TIMEOUT
    ops.set_wait_limit_ns(0)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    o = ops.attn_decode(q, k, v, r, w, 0, R, 0.1, lse=lse)
    assert ops.device_status(reset=True) == 0
    o_ref, lse_ref = O.attn_decode(q[:1].cpu(), k[:1].cpu(), v[:1].cpu(), r[:1].cpu(), w.cpu(), 0, R, 0.1)
    assert_bf16_close(o[:1], o_ref, lse[:1], lse_ref, "decode after a timed-out call")
