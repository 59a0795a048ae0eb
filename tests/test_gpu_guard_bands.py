"""Out-of-bounds writes, checked with guard bands (a bounds check that needs no
sanitizer).

Every output buffer of every entry point -- O, LSE, the decode workspaces, the
backward gradients and its workspace -- is placed in the middle of a larger
allocation whose bands before and after it hold a sentinel bit pattern.  After the
call the bands must still hold it, byte for byte, and the outputs themselves must
have been written everywhere (no sentinel left inside).  Shapes are ragged on
purpose: one token, a tile plus one row, a chunk starting mid-tile, odd group sizes,
short pages.
"""
import math

import pytest
import torch

from attention_learned_relative_b200 import ops, synth

pytestmark = pytest.mark.gpu

BAND = 4096            # bytes before and after each buffer (keeps 32-byte alignment)
SENTINEL = 0xA5        # byte pattern of the bands and of the buffer before the call


class Guarded:
    """A tensor view inside a sentinel-filled byte buffer with BAND bytes on each side."""

    def __init__(self, shape, dtype):
        esz = torch.empty((), dtype=dtype).element_size()
        n = 1
        for s in shape:
            n *= int(s)
        self.nbytes = n * esz
        self.raw = torch.full((BAND + self.nbytes + BAND,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[BAND:BAND + self.nbytes].view(dtype).view(*shape)

    def check(self, what, fully_written=True):
        torch.cuda.synchronize()
        raw = self.raw.cpu()
        assert bool((raw[:BAND] == SENTINEL).all()), what + ": write before the buffer"
        assert bool((raw[BAND + self.nbytes:] == SENTINEL).all()), what + ": write past the buffer"
        if fully_written and self.nbytes > 0:
            inner = raw[BAND:BAND + self.nbytes]
            esz = self.t.element_size()
            words = inner.view(-1, esz)
            untouched = (words == SENTINEL).all(dim=1)
            assert not bool(untouched.any()), what + ": %d elements never written" % int(untouched.sum())


@pytest.fixture(autouse=True)
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out"


def _x(B, T, Hq, Hkv, d, R, seed, dtype=torch.bfloat16, kv_T=None):
    kv_T = T if kv_T is None else kv_T
    return {
        "q": synth.normal((B, T, Hq, d), seed, "q", dtype=dtype, device="cuda"),
        "k": synth.normal((B, kv_T, Hkv, d), seed, "k", dtype=dtype, device="cuda"),
        "v": synth.normal((B, kv_T, Hkv, d), seed, "v", dtype=dtype, device="cuda"),
        "r": synth.normal((B, T, Hq), seed, "r", device="cuda"),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device="cuda"),
    }


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R", [
    (1, 1, 4, 2, 128, 0, 16),        # a single token
    (2, 129, 6, 2, 128, 0, 64),      # one tile plus one row, odd group (3)
    (1, 300, 8, 1, 64, 128, 128),    # windowed, d = 64, ragged tail
])
def test_prefill_writes_stay_inside(dtype, B, T, Hq, Hkv, d, window, R):
    x = _x(B, T, Hq, Hkv, d, R, seed=T + d, dtype=dtype)
    o = Guarded((B, T, Hq, d), dtype)
    lse = Guarded((B, Hq, T), torch.float32)
    ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, 1.0 / math.sqrt(d), out=o.t, lse=lse.t)
    o.check("o")
    lse.check("lse")


@pytest.mark.parametrize("T,q_off,kv_extra", [(100, 50, 0), (1, 127, 5), (130, 129, 300)])
def test_chunk_writes_stay_inside(T, q_off, kv_extra):
    B, Hq, Hkv, d, R = 2, 8, 2, 128, 256
    kv_T = q_off + T + kv_extra
    x = _x(B, T, Hq, Hkv, d, R, seed=q_off + T, kv_T=kv_T)
    o = Guarded((B, T, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq, T), torch.float32)
    ops.attn_fwd_chunk(x["q"], x["k"], x["v"], x["r"], x["w"], q_off, 0, R, 0.1, out=o.t, lse=lse.t)
    o.check("o")
    lse.check("lse")


def _dec_inputs(B, N, Hq, Hkv, d, R, seed):
    return {
        "q": synth.normal((B, Hq, d), seed, "q", dtype=torch.bfloat16, device="cuda"),
        "k": synth.normal((B, N, Hkv, d), seed, "k", dtype=torch.bfloat16, device="cuda"),
        "v": synth.normal((B, N, Hkv, d), seed, "v", dtype=torch.bfloat16, device="cuda"),
        "r": synth.normal((B, Hq), seed, "r", device="cuda"),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device="cuda"),
    }


@pytest.mark.parametrize("B,N,Hq,Hkv,window,R", [(3, 1, 8, 2, 0, 16), (2, 1000, 12, 3, 0, 300),
                                                 (1, 777, 8, 1, 256, 256)])
def test_decode_writes_stay_inside(B, N, Hq, Hkv, window, R):
    d = 128
    x = _dec_inputs(B, N, Hq, Hkv, d, R, seed=N)
    need = ops.decode_workspace_size(B, Hq, Hkv, N, d, window)
    ws = Guarded((need,), torch.uint8)
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ops.attn_decode(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, 0.1, out=o.t, lse=lse.t, workspace=ws.t)
    o.check("o")
    lse.check("lse")
    ws.check("workspace", fully_written=False)


def test_noalloc_decode_writes_stay_inside():
    B, N, Hq, Hkv, d, R = 2, 1000, 8, 2, 128, 64
    x = _dec_inputs(B, N, Hq, Hkv, d, R, seed=5)
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ops.attn_decode_noalloc(x["q"], x["k"], x["v"], x["r"], x["w"], 0, R, 0.1, out=o.t, lse=lse.t)
    o.check("o")
    lse.check("lse")


def test_paged_decode_writes_stay_inside():
    B, Hq, Hkv, d, R, page = 3, 8, 2, 128, 128, 64
    lens = [1, 65, 200]
    max_len = 256
    pages_per = max_len // page
    num_pages = B * pages_per
    kp = synth.normal((num_pages, page, Hkv, d), 7, "k", dtype=torch.bfloat16, device="cuda")
    vp = synth.normal((num_pages, page, Hkv, d), 7, "v", dtype=torch.bfloat16, device="cuda")
    table = torch.randperm(num_pages, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    table = table.reshape(B, pages_per).cuda()
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q = synth.normal((B, Hq, d), 7, "q", dtype=torch.bfloat16, device="cuda")
    r = synth.normal((B, Hq), 7, "r", device="cuda")
    w = synth.normal((Hq, R), 7, "w", std=0.5, device="cuda")
    need = ops.decode_paged_workspace_size(B, Hq, Hkv, max_len, d, 0)
    ws = Guarded((need,), torch.uint8)
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ops.attn_decode_paged(q, kp, vp, table, seq_lens, r, w, 0, R, max_len, 0.1, out=o.t, lse=lse.t, workspace=ws.t)
    o.check("o")
    lse.check("lse")
    ws.check("workspace", fully_written=False)


def test_bank_decode_writes_stay_inside():
    B, N, Hq, Hkv, d, R, C = 2, 900, 8, 2, 128, 200, 16
    x = _dec_inputs(B, N, Hq, Hkv, d, R, seed=11)
    rs = synth.normal((B, Hq, C), 11, "rs", std=0.25, device="cuda")
    proj = synth.normal((1, C, R), 11, "proj", std=0.5, device="cuda")
    need = ops.decode_bank_workspace_size(B, Hq, Hkv, N, d, 0, R)
    ws = Guarded((need,), torch.uint8)
    o = Guarded((B, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ops.attn_decode_bank(x["q"], x["k"], x["v"], rs, proj, 0, R, 0.1, out=o.t, lse=lse.t, workspace=ws.t)
    o.check("o")
    lse.check("lse")
    ws.check("workspace", fully_written=False)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,window", [(1, 0), (129, 0), (200, 64)])
def test_backward_writes_stay_inside(dtype, T, window):
    B, Hq, Hkv, d, R = 1, 6, 2, 64, 96
    x = _x(B, T, Hq, Hkv, d, R, seed=T + 1, dtype=dtype)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, 0.125, lse=lse)
    dout = synth.normal((B, T, Hq, d), 3, "bank", dtype=dtype, device="cuda")
    g = {"dq": Guarded((B, T, Hq, d), torch.float32), "dk": Guarded((B, T, Hkv, d), torch.float32),
         "dv": Guarded((B, T, Hkv, d), torch.float32), "dr": Guarded((B, T, Hq), torch.float32),
         "dw": Guarded((Hq, R), torch.float32)}
    ws = Guarded((int(ops.lib().relbias_attn_bwd_workspace_size(B, T, Hq)),), torch.uint8)
    ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, dout, window, R, 0.125, workspace=ws.t,
                 grads={n: gb.t for n, gb in g.items()})
    for n, gb in g.items():
        gb.check(n)
    ws.check("workspace", fully_written=False)


@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R,C,proj_heads", [
    (1, 1, 4, 2, 128, 0, 16, 3, 1),          # a single token
    (2, 129, 6, 2, 128, 0, 99, 16, 6),       # one tile plus one row, R not a multiple of 4
    (1, 300, 8, 1, 64, 128, 128, 5, 1),      # windowed, d = 64
])
def test_bank_prefill_writes_stay_inside(B, T, Hq, Hkv, d, window, R, C, proj_heads):
    x = _x(B, T, Hq, Hkv, d, R, seed=T + C)
    rs = synth.normal((B, T, Hq, C), T, "rs", std=0.25, device="cuda")
    proj = synth.normal((proj_heads, C, R), T, "proj", std=0.5, device="cuda")
    need = ops.fwd_bank_workspace_size(B, T, Hq, R, ops.RELBIAS_BF16)
    ws = Guarded((need,), torch.uint8)
    o = Guarded((B, T, Hq, d), torch.bfloat16)
    lse = Guarded((B, Hq, T), torch.float32)
    ops.attn_fwd_bank(x["q"], x["k"], x["v"], rs, proj, window, R, 1.0 / math.sqrt(d), out=o.t, lse=lse.t,
                      workspace=ws.t)
    o.check("o")
    lse.check("lse")
    ws.check("workspace", fully_written=False)


def test_bank_backward_writes_stay_inside():
    B, T, Hq, Hkv, d, R, C = 1, 200, 6, 2, 64, 77, 5
    x = _x(B, T, Hq, Hkv, d, R, seed=31)
    rs = synth.normal((B, T, Hq, C), 31, "rs", std=0.4, device="cuda")
    proj = synth.normal((1, C, R), 31, "proj", std=0.5, device="cuda")
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd_bank(x["q"], x["k"], x["v"], rs, proj, 64, R, 0.125, lse=lse)
    dout = synth.normal((B, T, Hq, d), 3, "bank", dtype=torch.bfloat16, device="cuda")
    g = {"dq": Guarded((B, T, Hq, d), torch.float32), "dk": Guarded((B, T, Hkv, d), torch.float32),
         "dv": Guarded((B, T, Hkv, d), torch.float32), "drs": Guarded((B, T, Hq, C), torch.float32),
         "dproj": Guarded((1, C, R), torch.float32)}
    ws = Guarded((int(ops.lib().relbias_attn_bwd_bank_workspace_size(B, T, Hq, R)),), torch.uint8)
    ops.attn_bwd_bank(x["q"], x["k"], x["v"], rs, proj, o, lse, dout, 64, R, 0.125, workspace=ws.t,
                      grads={n: gb.t for n, gb in g.items()})
    for n, gb in g.items():
        gb.check(n)
    ws.check("workspace", fully_written=False)
