"""The allocation-free decode entry point, relbias_attn_decode_noalloc.

It exists for callers that cannot allocate device memory -- for example a plugin
running inside an inference runtime that owns every device allocation, or a serving
loop that must not call cudaMalloc/cudaFree (cudaFree can synchronise the whole
device) between steps.  Instead of a caller-supplied workspace it uses scratch
compiled into the library.  These tests call it through the C ABI twice in a row,
on different inputs, and check that each result is bit-identical to the regular
entry point's (relbias_attn_decode with a caller workspace runs the same kernels
with the same split plan), and within the bf16 tolerance of a plain fp32
recomputation.  The file is named to be collected last.
"""
import ctypes
import math

import pytest
import torch

from attention_learned_relative_b200 import build, ops, synth
from parity import BF16_MAX_ABS, BF16_MEAN_ABS

pytestmark = pytest.mark.gpu


def _inputs(B, N, Hq, Hkv, d, R, seed):
    dev = "cuda"
    return {
        "q": synth.normal((B, Hq, d), seed, "q", dtype=torch.bfloat16, device=dev),
        "k": synth.normal((B, N, Hkv, d), seed, "k", dtype=torch.bfloat16, device=dev),
        "v": synth.normal((B, N, Hkv, d), seed, "v", dtype=torch.bfloat16, device=dev),
        "r": synth.normal((B, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
    }


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_call(lib, x, window, R, scale, o, lse, temp_n0=0):
    B, Hq, d = x["q"].shape
    _, N, Hkv, _ = x["k"].shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.relbias_attn_decode_noalloc(_p(x["q"]), _p(x["k"]), _p(x["v"]), _p(x["r"]), _p(x["w"]), _p(o),
                                           _p(lse), B, N, Hq, Hkv, d, window, R, scale, temp_n0, ops.RELBIAS_BF16,
                                           stream)


def _check_against_regular(lib, B, N, Hq, Hkv, d, R, window, temp_n0, seeds):
    """Calls in a row through the C ABI, each on fresh inputs, each compared with
    relbias_attn_decode given a caller workspace.  Both run the same kernels with the
    same split plan, so the results must be bit-identical."""
    scale = 1.0 / math.sqrt(d)
    for call, seed in enumerate(seeds):
        x = _inputs(B, N, Hq, Hkv, d, R, seed)
        lse_ref = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        o_ref = ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, scale, lse=lse_ref,
                                temp_n0=temp_n0)
        o = torch.full_like(x["q"], float("nan"))
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        rc = _noalloc_call(lib, x, window, R, scale, o, lse, temp_n0)
        assert rc == ops.RELBIAS_OK, ops.last_error()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), "call %d: output differs from relbias_attn_decode" % call
        assert torch.equal(lse, lse_ref), "call %d: lse differs from relbias_attn_decode" % call
        # And both are right: the regular entry point's parity bound against nothing but
        # itself is not enough, so hold the pair to the bf16 tolerance of a plain
        # fp32 recomputation of the last row's softmax attention.
        err = (o.float() - _fp32_decode(x, window, R, scale, temp_n0)).abs()
        assert err.max().item() <= BF16_MAX_ABS and err.mean().item() <= BF16_MEAN_ABS, "call %d" % call


def _fp32_decode(x, window, R, scale, temp_n0):
    """Plain fp32 torch recomputation of the decode step (a sanity bound only)."""
    q = x["q"].float()
    B, Hq, d = q.shape
    k, v = x["k"].float(), x["v"].float()
    N, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    lo = max(0, N - window) if window > 0 else 0
    kk = k[:, lo:].repeat_interleave(G, dim=2)            # [B, n, Hq, d]
    vv = v[:, lo:].repeat_interleave(G, dim=2)
    s = torch.einsum("bhd,bjhd->bhj", q, kk) * scale
    dist = (N - 1) - torch.arange(lo, N, device=q.device)
    wd = torch.zeros(Hq, N - lo, device=q.device)
    inside = dist < R
    wd[:, inside] = x["w"][:, dist[inside]]
    s = s + x["r"][:, :, None] * wd[None]
    n = N - lo
    if temp_n0 > 1 and n > temp_n0:
        s = s * (math.log(n) / math.log(temp_n0))
    p = torch.softmax(s, dim=-1)
    return torch.einsum("bhj,bjhd->bhd", p, vv)


def test_noalloc_decode_matches_regular_entry_point_twice():
    build.build()
    lib = ops.lib()
    ops.device_status(reset=True)
    B, N, Hq, Hkv, d, R = 4, 50000, 32, 4, 128, 1024
    assert 0 < ops.decode_workspace_size(B, Hq, Hkv, N, d, 0) <= 8 << 20
    _check_against_regular(lib, B, N, Hq, Hkv, d, R, 0, 0, (101, 202))
    assert ops.device_status(reset=True) == 0


def test_noalloc_windowed_decode_with_temperature():
    build.build()
    lib = ops.lib()
    ops.device_status(reset=True)
    # The local-layer shape: a 512-key window with the bias over all of it, and a
    # context-length temperature that is active (the window holds n = 512 > 300 keys).
    _check_against_regular(lib, 2, 3000, 32, 4, 128, 512, 512, 300, (303, 404))
    assert ops.device_status(reset=True) == 0


def test_noalloc_decode_just_under_the_scratch_limit():
    build.build()
    lib = ops.lib()
    ops.device_status(reset=True)
    # 496 sequences x 4 key/value heads = 1984 (sequence, head) pairs: one split each,
    # 496 x 32 records of 528 bytes = 8,380,416 bytes, just under the 8 MiB scratch.
    B, N, Hq, Hkv, d, R = 496, 64, 32, 4, 128, 48
    need = ops.decode_workspace_size(B, Hq, Hkv, N, d, 0)
    assert (8 << 20) - 16384 < need <= 8 << 20, need
    _check_against_regular(lib, B, N, Hq, Hkv, d, R, 0, 0, (505, 606))
    assert ops.device_status(reset=True) == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    build.build()
    lib = ops.lib()
    # 2048 (sequence, key/value head) pairs: one split each, 256 x 64 partial records
    # of 528 bytes = 8.65 MB, beyond the 8 MiB scratch.
    B, N, Hq, Hkv, d, R = 256, 64, 64, 8, 128, 16
    need = ops.decode_workspace_size(B, Hq, Hkv, N, d, 0)
    assert need > 8 << 20
    x = {"q": torch.zeros(B, Hq, d, dtype=torch.bfloat16, device="cuda"),
         "k": torch.zeros(B, N, Hkv, d, dtype=torch.bfloat16, device="cuda"),
         "r": torch.zeros(B, Hq, device="cuda"), "w": torch.zeros(Hq, R, device="cuda")}
    x["v"] = x["k"]
    o = torch.empty_like(x["q"])
    lse = torch.empty(B, Hq, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.relbias_attn_decode_noalloc(_p(x["q"]), _p(x["k"]), _p(x["v"]), _p(x["r"]), _p(x["w"]), _p(o),
                                         _p(lse), B, N, Hq, Hkv, d, 0, R, 0.1, 0, ops.RELBIAS_BF16, stream)
    assert rc == ops.RELBIAS_ERR_UNSUPPORTED
    assert "static scratch" in ops.last_error()
