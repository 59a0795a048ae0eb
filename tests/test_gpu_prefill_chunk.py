"""GPU parity of chunked prefill (relbias_attn_fwd_chunk): T query rows at positions
q_off ... q_off+T-1 against a cache holding the prefix and the chunk's own keys.

Cache rows past the chunk are filled with NaN (stale rows of a serving cache), so a
kernel that let them into a product would fail.  The oracle computes the same rows
of the whole sequence.
"""
import math

import pytest
import torch

from attention_learned_relative_b200 import ops, synth
from oracle import oracle as O
from parity import assert_bf16_close, assert_fp32_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out"


def _seq(B, L, Hq, Hkv, d, R, seed, dtype, extra):
    dev = "cuda"
    x = {
        "q": synth.normal((B, L, Hq, d), seed, "q", dtype=dtype, device=dev),
        "k": synth.normal((B, L, Hkv, d), seed, "k", dtype=dtype, device=dev),
        "v": synth.normal((B, L, Hkv, d), seed, "v", dtype=dtype, device=dev),
        "r": synth.normal((B, L, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
    }
    # the cache: the sequence's L rows, then `extra` stale rows
    kc = torch.full((B, L + extra, Hkv, d), float("nan"), dtype=dtype, device=dev)
    vc = torch.full_like(kc, float("nan"))
    kc[:, :L] = x["k"]
    vc[:, :L] = x["v"]
    x["kc"], x["vc"] = kc, vc
    return x


CASES = [
    # dtype,          B, q_off, T,   Hq, Hkv, d,   window, R,   temp_n0
    (torch.bfloat16, 1, 0, 300, 8, 2, 128, 0, 64, 0),
    (torch.bfloat16, 1, 1, 200, 8, 2, 128, 0, 128, 0),           # diagonal one row into a tile
    (torch.bfloat16, 2, 127, 130, 8, 2, 128, 0, 300, 0),
    (torch.bfloat16, 1, 128, 128, 8, 1, 128, 512, 512, 0),       # local layer, aligned chunk
    (torch.bfloat16, 1, 300, 257, 4, 2, 128, 512, 512, 0),       # local layer, unaligned
    (torch.bfloat16, 1, 1000, 100, 4, 1, 128, 0, 1024, 600),     # global layer, temperature
    (torch.bfloat16, 1, 5, 1, 8, 2, 128, 0, 16, 0),              # one query row
    (torch.bfloat16, 1, 700, 64, 6, 2, 64, 128, 100, 0),         # head dim 64, GQA group 3
    (torch.float32, 1, 50, 60, 4, 2, 64, 0, 32, 0),
    (torch.float32, 2, 33, 40, 4, 1, 128, 16, 20, 30),
]


@pytest.mark.parametrize("dtype,B,q_off,T,Hq,Hkv,d,window,R,temp_n0", CASES)
def test_chunk_parity(dtype, B, q_off, T, Hq, Hkv, d, window, R, temp_n0):
    L = q_off + T
    x = _seq(B, L, Hq, Hkv, d, R, seed=q_off + 3 * T + R, dtype=dtype, extra=77)
    scale = 1.0 / math.sqrt(d)
    q = x["q"][:, q_off:].contiguous()
    r = x["r"][:, q_off:].contiguous()
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd_chunk(q, x["kc"], x["vc"], r, x["w"], q_off, window, R, scale, lse=lse, temp_n0=temp_n0)
    torch.cuda.synchronize()
    rows = [(b, h, q_off + i) for b in range(B) for h in range(Hq) for i in range(T)]
    o_ref, lse_ref = O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), window, R,
                                    scale, rows=rows, temp_n0=temp_n0)
    o_rows = o.permute(0, 2, 1, 3).reshape(-1, d)          # (b, h, i) order, as `rows`
    lse_rows = lse.reshape(-1)
    check = assert_fp32_close if dtype == torch.float32 else assert_bf16_close
    check(o_rows, o_ref, lse_rows, lse_ref, "chunk %s" % ((dtype, B, q_off, T, window, R, temp_n0),))


def test_chunk_at_zero_is_the_whole_sequence_bitwise():
    x = _seq(2, 333, 8, 2, 128, 128, seed=3, dtype=torch.bfloat16, extra=0)
    o1 = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], 0, 128, 0.09)
    o2 = ops.attn_fwd_chunk(x["q"], x["k"], x["v"], x["r"], x["w"], 0, 0, 128, 0.09)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_chunk_rejects_a_cache_shorter_than_the_chunk():
    x = _seq(1, 100, 4, 2, 128, 16, seed=4, dtype=torch.bfloat16, extra=0)
    with pytest.raises(ops.RelbiasError):
        ops.attn_fwd_chunk(x["q"][:, 50:].contiguous(), x["k"][:, :120].contiguous(), x["v"][:, :120].contiguous(),
                           x["r"][:, 50:].contiguous(), x["w"], 80, 0, 16)   # 80 + 50 > 120
