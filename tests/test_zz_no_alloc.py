"""The allocation-free decode entry point, relbias_attn_decode_noalloc.

It exists for callers that cannot allocate device memory -- for example a plugin
running inside an inference runtime that owns every device allocation, or a serving
loop that must not call cudaMalloc/cudaFree (cudaFree can synchronise the whole
device) between steps.  Instead of a caller-supplied workspace it uses scratch
compiled into the library.  These tests call it through the C ABI twice in a row,
on different inputs, and check each result against the regular entry point
(relbias_attn_decode with a caller workspace) within the bf16 tolerance of the
other parity tests.  The file is named to be collected last.
"""
import ctypes
import math

import pytest
import torch

from attention_learned_relative_b200 import build, ops, synth
from parity import BF16_LSE_ABS, BF16_MAX_ABS, BF16_MEAN_ABS

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


def _noalloc_call(lib, x, window, R, scale, o, lse):
    B, Hq, d = x["q"].shape
    _, N, Hkv, _ = x["k"].shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.relbias_attn_decode_noalloc(_p(x["q"]), _p(x["k"]), _p(x["v"]), _p(x["r"]), _p(x["w"]), _p(o),
                                           _p(lse), B, N, Hq, Hkv, d, window, R, scale, 0, ops.RELBIAS_BF16, stream)


def test_noalloc_decode_matches_regular_entry_point_twice():
    build.build()
    lib = ops.lib()
    ops.device_status(reset=True)
    B, N, Hq, Hkv, d, R = 4, 50000, 32, 4, 128, 1024
    scale = 1.0 / math.sqrt(d)
    assert 0 < ops.decode_workspace_size(B, Hq, Hkv, N, d, 0) <= 8 << 20
    for call, seed in enumerate((101, 202)):          # two calls in a row, different inputs
        x = _inputs(B, N, Hq, Hkv, d, R, seed)
        lse_ref = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        o_ref = ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], 0, R, scale, lse=lse_ref)
        o = torch.empty_like(x["q"])
        lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        rc = _noalloc_call(lib, x, 0, R, scale, o, lse)
        assert rc == ops.RELBIAS_OK, ops.last_error()
        torch.cuda.synchronize()
        err = (o.float() - o_ref.float()).abs()
        assert err.max().item() <= BF16_MAX_ABS and err.mean().item() <= BF16_MEAN_ABS, "call %d" % call
        assert (lse - lse_ref).abs().max().item() <= BF16_LSE_ABS, "call %d" % call
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
