"""GPU parity of the shared-bank bias against the fp64 oracle.

The essay's recipe keeps a bank of C functions of distance shared by the heads of a
layer, and gives each token and head C coefficients; the bias is their product
("Thinking Machines dropped RoPE", steps 1-2).  relbias_attn_fwd_bank runs it on the
fp32 prefill path and on the bf16 tensor-core prefill (through per-row curves),
relbias_attn_decode_bank on the bf16 split-KV decode (through per-(sequence, head)
curves).  The oracle takes the same rs [.., C] and proj
[1 or Hq, C, R] tensors.
"""
import math

import numpy as np
import pytest
import torch

from attention_learned_relative_b200 import ops, synth
from attention_learned_relative_b200.workloads import WORKLOADS, make_inputs
from oracle import oracle as O
from parity import assert_bf16_close, assert_fp32_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out"


PREFILL_CASES = [
    # B, T,   Hq, Hkv, d,   window, R,   C,  proj_heads, temp_n0
    (1, 200, 4, 2, 64, 0, 64, 16, 1, 0),        # the essay's 16-function bank, shared
    (2, 150, 4, 1, 32, 48, 40, 4, 4, 0),        # a bank per head, windowed
    (1, 300, 2, 2, 128, 0, 100, 7, 1, 50),      # temperature
    (1, 130, 8, 2, 256, 0, 130, 1, 1, 0),       # one shared function
]


@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R,C,proj_heads,temp_n0", PREFILL_CASES)
def test_fp32_prefill_bank_parity(B, T, Hq, Hkv, d, window, R, C, proj_heads, temp_n0):
    seed = T + 3 * C + d
    dev = "cuda"
    q = synth.normal((B, T, Hq, d), seed, "q", device=dev)
    k = synth.normal((B, T, Hkv, d), seed, "k", device=dev)
    v = synth.normal((B, T, Hkv, d), seed, "v", device=dev)
    rs = synth.normal((B, T, Hq, C), seed, "rs", std=1.0 / math.sqrt(C), device=dev)
    proj = synth.normal((proj_heads, C, R), seed, "proj", std=0.5, device=dev)
    scale = 1.0 / math.sqrt(d)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device=dev)
    o = ops.attn_fwd_bank(q, k, v, rs, proj, window, R, scale, lse=lse, temp_n0=temp_n0)
    torch.cuda.synchronize()
    o_ref, lse_ref = O.attn_prefill(q.cpu(), k.cpu(), v.cpu(), rs.cpu(), proj.cpu(), window, R, scale,
                                    temp_n0=temp_n0)
    assert_fp32_close(o, o_ref, lse, lse_ref, "fp32 bank %s" % ((B, T, Hq, Hkv, d, window, R, C, proj_heads),))


def test_fp32_bank_of_one_function_per_head_is_the_rank1_form_bitwise():
    """C = 1 with a bank per head is the rank-1 form: same arithmetic, same bits."""
    B, T, Hq, Hkv, d, R = 2, 100, 4, 2, 64, 50
    dev = "cuda"
    q = synth.normal((B, T, Hq, d), 9, "q", device=dev)
    k = synth.normal((B, T, Hkv, d), 9, "k", device=dev)
    v = synth.normal((B, T, Hkv, d), 9, "v", device=dev)
    r = synth.normal((B, T, Hq), 9, "r", device=dev)
    w = synth.normal((Hq, R), 9, "w", std=0.5, device=dev)
    o1 = ops.attn_fwd(q, k, v, r, w, 0, R, 0.125)
    o2 = ops.attn_fwd_bank(q, k, v, r[..., None].contiguous(), w[:, None, :].contiguous(), 0, R, 0.125)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


BF16_CASES = [
    # B, T,   Hq, Hkv, d,   window, R,   C,  proj_heads, temp_n0
    (1, 200, 4, 2, 128, 0, 64, 16, 1, 0),       # the essay's 16-function bank, shared; ragged tail
    (2, 300, 8, 2, 128, 128, 128, 16, 8, 0),    # a bank per head, windowed (local-layer form)
    (1, 513, 6, 3, 64, 0, 300, 5, 1, 100),      # odd group, d = 64, temperature, R not a tile multiple
    (1, 1, 4, 4, 128, 0, 16, 3, 1, 0),          # a single token
    (1, 260, 4, 2, 128, 0, 1000, 16, 1, 0),     # R beyond the sequence
    (1, 150, 4, 2, 128, 0, 77, 7, 4, 0),        # R odd (the curve kernel's scalar loads)
]


def _bank_inputs(B, T, Hq, Hkv, d, R, C, proj_heads, seed, dtype=torch.bfloat16):
    dev = "cuda"
    return (synth.normal((B, T, Hq, d), seed, "q", dtype=dtype, device=dev),
            synth.normal((B, T, Hkv, d), seed, "k", dtype=dtype, device=dev),
            synth.normal((B, T, Hkv, d), seed, "v", dtype=dtype, device=dev),
            synth.normal((B, T, Hq, C), seed, "rs", std=1.0 / math.sqrt(C), device=dev),
            synth.normal((proj_heads, C, R), seed, "proj", std=0.5, device=dev))


@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R,C,proj_heads,temp_n0", BF16_CASES)
def test_bf16_prefill_bank_parity(B, T, Hq, Hkv, d, window, R, C, proj_heads, temp_n0):
    """The tensor-core prefill with the bank's per-row curves, against the oracle's bank form."""
    q, k, v, rs, proj = _bank_inputs(B, T, Hq, Hkv, d, R, C, proj_heads, seed=T + C + d)
    scale = 1.0 / math.sqrt(d)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd_bank(q, k, v, rs, proj, window, R, scale, lse=lse, temp_n0=temp_n0)
    torch.cuda.synchronize()
    o_ref, lse_ref = O.attn_prefill(q.cpu(), k.cpu(), v.cpu(), rs.cpu(), proj.cpu(), window, R, scale,
                                    temp_n0=temp_n0)
    assert_bf16_close(o, o_ref, lse, lse_ref, "bf16 bank %s" % ((B, T, Hq, Hkv, d, window, R, C, proj_heads),))


def test_bf16_bank_of_one_function_per_head_matches_rank1():
    """C = 1 with a bank per head is the rank-1 form; the two bf16 paths agree to rounding
    (the bank path forms r * w in its curve kernel, the rank-1 path in the softmax)."""
    B, T, Hq, Hkv, d, R = 2, 300, 8, 2, 128, 200
    dev = "cuda"
    q = synth.normal((B, T, Hq, d), 12, "q", dtype=torch.bfloat16, device=dev)
    k = synth.normal((B, T, Hkv, d), 12, "k", dtype=torch.bfloat16, device=dev)
    v = synth.normal((B, T, Hkv, d), 12, "v", dtype=torch.bfloat16, device=dev)
    r = synth.normal((B, T, Hq), 12, "r", device=dev)
    w = synth.normal((Hq, R), 12, "w", std=0.5, device=dev)
    l1 = torch.empty(B, Hq, T, dtype=torch.float32, device=dev)
    l2 = torch.empty_like(l1)
    o1 = ops.attn_fwd(q, k, v, r, w, 128, R, 0.09, lse=l1)
    o2 = ops.attn_fwd_bank(q, k, v, r[..., None].contiguous(), w[:, None, :].contiguous(), 128, R, 0.09, lse=l2)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1.6e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_bf16_bank_unaligned_proj_matches_aligned():
    """proj at a 4-byte offset (not 16-byte aligned) takes the curve kernel's scalar
    loads and gives the same output, bit for bit."""
    B, T, Hq, Hkv, d, R, C = 1, 300, 4, 2, 128, 256, 16
    q, k, v, rs, proj = _bank_inputs(B, T, Hq, Hkv, d, R, C, 1, seed=17)
    buf = torch.empty(proj.numel() + 1, dtype=torch.float32, device="cuda")
    shifted = buf[1:].view(proj.shape)
    shifted.copy_(proj)
    assert shifted.data_ptr() % 16 != 0 and shifted.is_contiguous()
    o1 = ops.attn_fwd_bank(q, k, v, rs, proj, 0, R, 0.1)
    o2 = ops.attn_fwd_bank(q, k, v, rs, shifted, 0, R, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_bf16_bank_workspace_is_not_read_before_written():
    """The curve workspace's prior contents do not matter (NaN-filled here)."""
    B, T, Hq, Hkv, d, R, C = 1, 257, 4, 2, 128, 100, 16
    q, k, v, rs, proj = _bank_inputs(B, T, Hq, Hkv, d, R, C, 1, seed=77)
    need = ops.fwd_bank_workspace_size(B, T, Hq, R, ops.RELBIAS_BF16)
    ws = torch.full((need // 4,), float("nan"), dtype=torch.float32, device="cuda").view(torch.uint8)
    o = ops.attn_fwd_bank(q, k, v, rs, proj, 0, R, 0.1, workspace=ws)
    torch.cuda.synchronize()
    o_ref, _ = O.attn_prefill(q.cpu(), k.cpu(), v.cpu(), rs.cpu(), proj.cpu(), 0, R, 0.1)
    assert_bf16_close(o, o_ref, what="bf16 bank, NaN-filled workspace")


def test_bf16_prefill_bank_workload_sampled():
    """The local-layer shape with the essay's 16-function shared bank, in the launch
    configuration the benchmark times, on sampled rows."""
    from parity import sample_rows
    wl = WORKLOADS["local_prefill_bank_bf16"]
    x = make_inputs(wl, device="cuda")
    B, T, Hq, d = x["q"].shape
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], wl.window, wl.R, wl.scale, lse=lse)
    torch.cuda.synchronize()
    rows = sample_rows(B, T, Hq, per_head=3, seed=5, extra=(8190,))
    o_ref, lse_ref = O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["rs"].cpu(), x["proj"].cpu(),
                                    wl.window, wl.R, wl.scale, rows=rows)
    got = o.float().cpu()[rows[:, 0], rows[:, 2], rows[:, 1]]
    got_lse = lse.cpu()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_bf16_close(got, o_ref, got_lse, lse_ref, wl.name)


DECODE_CASES = [
    # B, N,    Hq, Hkv, window, R,    C,  proj_heads, temp_n0
    (2, 3000, 8, 2, 0, 1024, 16, 1, 0),
    (1, 5000, 16, 4, 512, 512, 4, 16, 0),     # a bank per head, windowed
    (3, 700, 8, 1, 0, 300, 9, 1, 200),        # group of 8, temperature
    (2, 40, 8, 2, 0, 2000, 16, 1, 0),         # R beyond the cache
]


@pytest.mark.parametrize("B,N,Hq,Hkv,window,R,C,proj_heads,temp_n0", DECODE_CASES)
def test_decode_bank_parity(B, N, Hq, Hkv, window, R, C, proj_heads, temp_n0):
    d, dev = 128, "cuda"
    seed = N + C
    q = synth.normal((B, Hq, d), seed, "q", dtype=torch.bfloat16, device=dev)
    k = synth.normal((B, N, Hkv, d), seed, "k", dtype=torch.bfloat16, device=dev)
    v = synth.normal((B, N, Hkv, d), seed, "v", dtype=torch.bfloat16, device=dev)
    rs = synth.normal((B, Hq, C), seed, "rs", std=1.0 / math.sqrt(C), device=dev)
    proj = synth.normal((proj_heads, C, R), seed, "proj", std=0.5, device=dev)
    scale = 1.0 / math.sqrt(d)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    o = ops.attn_decode_bank(q, k, v, rs, proj, window, R, scale, lse=lse, temp_n0=temp_n0)
    torch.cuda.synchronize()
    o_ref, lse_ref = O.attn_decode(q.cpu(), k.cpu(), v.cpu(), rs.cpu(), proj.cpu(), window, R, scale,
                                   temp_n0=temp_n0)
    assert_bf16_close(o, o_ref, lse, lse_ref, "decode bank %s" % ((B, N, Hq, Hkv, window, R, C, proj_heads),))


def test_decode_bank_of_one_function_per_head_matches_rank1():
    """C = 1 with a bank per head gives the rank-1 decode up to the rounding of the
    precomputed curve r*w (one fp32 product) against the in-kernel fused multiply-add."""
    B, N, Hq, Hkv, d, R = 2, 2000, 8, 2, 128, 512
    x = {"q": synth.normal((B, Hq, d), 4, "q", dtype=torch.bfloat16, device="cuda"),
         "k": synth.normal((B, N, Hkv, d), 4, "k", dtype=torch.bfloat16, device="cuda"),
         "v": synth.normal((B, N, Hkv, d), 4, "v", dtype=torch.bfloat16, device="cuda"),
         "r": synth.normal((B, Hq), 4, "r", device="cuda"),
         "w": synth.normal((Hq, R), 4, "w", std=0.5, device="cuda")}
    o1 = ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], 0, R, 0.09)
    o2 = ops.attn_decode_bank(x["q"], x["k"], x["v"], x["r"][..., None].contiguous(), x["w"][:, None, :].contiguous(),
                              0, R, 0.09)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 4e-3


def test_decode_bank_workload_sampled():
    """The 8 x 1,048,576-row bank workload in the benchmark's launch configuration,
    checked on sampled (sequence, key/value head) groups against the oracle on the
    group's full cache slice."""
    wl = WORKLOADS["global_decode_bank_bf16"]
    x = make_inputs(wl, device="cuda")
    B, Hq, d = x["q"].shape
    N = wl.T
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    ws = torch.empty(ops.decode_bank_workspace_size(B, Hq, wl.Hkv, N, d, wl.window, wl.R), dtype=torch.uint8,
                     device="cuda")
    o = ops.attn_decode_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], wl.window, wl.R, wl.scale, lse=lse,
                             workspace=ws)
    torch.cuda.synchronize()
    G = wl.group
    for (b, g) in [(1, 2), (7, 0)]:
        heads = list(range(g * G, (g + 1) * G))
        k_sl = x["k"][b:b + 1, :, g:g + 1, :].cpu()
        v_sl = x["v"][b:b + 1, :, g:g + 1, :].cpu()
        req = np.array([(0, hl, N - 1) for hl in range(G)], dtype=np.int64)
        o_ref, lse_ref = O.attn_rows(x["q"][b, heads].float().cpu(), x["rs"][b, heads].cpu(), x["proj"].cpu(),
                                     k_sl, v_sl, req, G, wl.window, wl.R, wl.scale)
        assert_bf16_close(o[b, heads], o_ref, lse[b, heads], lse_ref, "decode bank workload (b=%d, g=%d)" % (b, g))
