"""GPU parity of the decode entry point (relbias_attn_decode) against the fp64 oracle.

One query per sequence at position n_ctx-1 against a bf16 cache.  Small caches are
checked on every output; the 1,048,576-row workload runs in the benchmark's launch
configuration and is checked on sampled (sequence, key/value head) groups, each
against the oracle on that group's full cache slice.
"""
import math

import numpy as np
import pytest
import torch

from attention_learned_relative_b200 import ops, synth
from attention_learned_relative_b200.workloads import WORKLOADS, make_inputs
from oracle import oracle as O
from parity import assert_bf16_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out"


def _inputs(B, N, Hq, Hkv, d, R, seed):
    dev = "cuda"
    return {
        "q": synth.normal((B, Hq, d), seed, "q", dtype=torch.bfloat16, device=dev),
        "k": synth.normal((B, N, Hkv, d), seed, "k", dtype=torch.bfloat16, device=dev),
        "v": synth.normal((B, N, Hkv, d), seed, "v", dtype=torch.bfloat16, device=dev),
        "r": synth.normal((B, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
    }


def _run(x, window, R, scale):
    B, Hq, _ = x["q"].shape
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    o = ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, scale, lse=lse)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("B,N,Hq,Hkv,window,R,n0", [
    (2, 3000, 8, 2, 0, 512, 1000),     # tau = ln 3000 / ln 1000
    (1, 5000, 16, 4, 512, 512, 100),   # windowed: the query sees 512 keys
])
def test_decode_context_length_temperature(B, N, Hq, Hkv, window, R, n0):
    x = _inputs(B, N, Hq, Hkv, 128, R, seed=N + n0)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    o = ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, 0.0884, lse=lse, temp_n0=n0)
    torch.cuda.synchronize()
    o_ref, lse_ref = O.attn_decode(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), window, R,
                                   0.0884, temp_n0=n0)
    assert_bf16_close(o, o_ref, lse, lse_ref, "decode temperature %s" % ((B, N, Hq, Hkv, window, R, n0),))


DECODE_CASES = [
    # B, N,     Hq, Hkv, window, R
    (2, 1, 8, 1, 0, 16),          # cache holds only the query's own row
    (2, 31, 8, 2, 0, 16),         # less than one chunk
    (3, 1000, 8, 1, 0, 64),       # ragged last chunk
    (2, 4096, 32, 4, 0, 1024),    # the global-layer head layout
    (1, 5000, 16, 4, 512, 512),   # local layer: window 512
    (2, 3000, 4, 4, 0, 100),      # GQA group 1
    (1, 2500, 12, 3, 0, 2500),    # group 4, bias over the whole cache
    (2, 777, 8, 2, 0, 0),         # R = 0
]


@pytest.mark.parametrize("B,N,Hq,Hkv,window,R", DECODE_CASES)
def test_decode_parity(B, N, Hq, Hkv, window, R):
    d = 128
    x = _inputs(B, N, Hq, Hkv, d, R, seed=N + R)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(x, window, R, scale)
    o_ref, lse_ref = O.attn_decode(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), window,
                                   R, scale)
    assert_bf16_close(o, o_ref, lse, lse_ref, "decode %s" % ((B, N, Hq, Hkv, window, R),))


def test_decode_matches_last_prefill_row():
    """Decode against n_ctx rows equals the last row of a prefill over the same
    n_ctx tokens (both checked against the oracle, and against each other)."""
    B, N, Hq, Hkv, d, R = 1, 1500, 8, 2, 128, 600
    seed = 77
    q_all = synth.normal((B, N, Hq, d), seed, "q", dtype=torch.bfloat16, device="cuda")
    k = synth.normal((B, N, Hkv, d), seed, "k", dtype=torch.bfloat16, device="cuda")
    v = synth.normal((B, N, Hkv, d), seed, "v", dtype=torch.bfloat16, device="cuda")
    r_all = synth.normal((B, N, Hq), seed, "r", device="cuda")
    w = synth.normal((Hq, R), seed, "w", std=0.5, device="cuda")
    o_pre = ops.attn_fwd(q_all, k, v, r_all, w, 0, R, 0.1)
    o_dec = ops.attn_decode(q_all[:, -1].contiguous(), k, v, r_all[:, -1].contiguous(), w, 0, R, 0.1)
    torch.cuda.synchronize()
    assert (o_pre[:, -1].float() - o_dec.float()).abs().max().item() <= 2e-2


def test_decode_split_invariance():
    """The same cache seen through different split counts (more sequences change the
    number of CTAs per sequence) gives the same answer within rounding."""
    N, Hq, Hkv, d, R = 20000, 8, 1, 128, 1024
    x = _inputs(1, N, Hq, Hkv, d, R, seed=5)
    o1, l1 = _run(x, 0, R, 0.1)
    # Replicate the sequence 6 times: fewer splits per sequence.
    x6 = {k_: torch.cat([t] * 6, dim=0).contiguous() if k_ != "w" else t for k_, t in x.items()}
    o6, l6 = _run(x6, 0, R, 0.1)
    assert (o6.float() - o1.float()).abs().max().item() <= 4e-3
    assert (l6 - l1).abs().max().item() <= 1e-4


def test_decode_workload_sampled():
    wl = WORKLOADS["global_decode_bf16"]
    x = make_inputs(wl, device="cuda")
    B, Hq, d = x["q"].shape
    N = wl.T
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    o = ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], wl.window, wl.R, wl.scale, lse=lse)
    torch.cuda.synchronize()
    G = wl.group
    for (b, g) in [(0, 0), (5, 3)]:
        heads = list(range(g * G, (g + 1) * G))
        k_sl = x["k"][b:b + 1, :, g:g + 1, :].cpu()
        v_sl = x["v"][b:b + 1, :, g:g + 1, :].cpu()
        req = np.array([(0, hl, N - 1) for hl in range(G)], dtype=np.int64)
        o_ref, lse_ref = O.attn_rows(x["q"][b, heads].float().cpu(), x["r"][b, heads].cpu().reshape(G, 1),
                                     x["w"][heads].cpu().reshape(G, 1, wl.R), k_sl, v_sl, req, G, wl.window, wl.R,
                                     wl.scale)
        assert_bf16_close(o[b, heads], o_ref, lse[b, heads], lse_ref, "decode workload (b=%d, g=%d)" % (b, g))


def test_decode_small_group_reads_only_its_own_features():
    """Group size 4 (fewer query heads than the kernel's 8 head columns): the padding
    columns must not read r.  r sits at the very end of a buffer whose next elements
    are NaN; reading them would still leave O finite, so the check here is that the
    result equals the same call with r in a buffer of its own, bit for bit."""
    B, N, Hq, Hkv, d, R = 3, 700, 8, 2, 128, 256
    x = _inputs(B, N, Hq, Hkv, d, R, seed=4242)
    o_ref, lse_ref = _run(x, 0, R, 0.1)
    buf = torch.full((B * Hq + 64,), float("nan"), dtype=torch.float32, device="cuda")
    buf[:B * Hq] = x["r"].reshape(-1)
    x_tail = dict(x, r=buf[:B * Hq].view(B, Hq))
    o, lse = _run(x_tail, 0, R, 0.1)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    o_or, lse_or = O.attn_decode(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), 0, R, 0.1)
    assert_bf16_close(o, o_or, lse, lse_or, "decode group 4")
