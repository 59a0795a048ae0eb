"""GPU parity of the paged, variable-length decode (relbias_attn_decode_paged).

Each sequence's cache is drawn contiguously, scattered into shuffled pages of a pool
whose other pages hold NaN (so a stray read shows), and the kernel's output is
compared with the fp64 oracle's decode on that sequence's own contiguous cache.
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
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel reported a bad status"


def _paged_inputs(lens, Hq, Hkv, R, page_size, seed, d=128, spare_pages=3, max_seq_len=None):
    """Per-sequence caches [n_b, Hkv, d] scattered into a shuffled page pool.  The block
    table has room for max_seq_len rows per sequence (unused entries hold -7)."""
    dev = "cuda"
    B = len(lens)
    caches_k = [synth.normal((n, Hkv, d), seed + 11 * b, "k", dtype=torch.bfloat16, device=dev)
                for b, n in enumerate(lens)]
    caches_v = [synth.normal((n, Hkv, d), seed + 11 * b, "v", dtype=torch.bfloat16, device=dev)
                for b, n in enumerate(lens)]
    blocks = [(n + page_size - 1) // page_size for n in lens]
    max_pages = max(max(blocks), ((max_seq_len or 0) + page_size - 1) // page_size)
    num_pages = sum(blocks) + spare_pages
    perm = np.random.default_rng(seed).permutation(num_pages)
    pool_k = torch.full((num_pages, page_size, Hkv, d), float("nan"), dtype=torch.bfloat16, device=dev)
    pool_v = torch.full_like(pool_k, float("nan"))
    table = torch.full((B, max_pages), -7, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(lens):
        for blk in range(blocks[b]):
            pg = int(perm[nxt])
            nxt += 1
            table[b, blk] = pg
            rows = slice(blk * page_size, min(n, (blk + 1) * page_size))
            cnt = rows.stop - rows.start
            pool_k[pg, :cnt] = caches_k[b][rows]
            pool_v[pg, :cnt] = caches_v[b][rows]
    x = {
        "q": synth.normal((B, Hq, d), seed, "q", dtype=torch.bfloat16, device=dev),
        "r": synth.normal((B, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
        "k_pages": pool_k, "v_pages": pool_v,
        "table": table.to(dev), "lens": torch.tensor(lens, dtype=torch.int32, device=dev),
        "caches_k": caches_k, "caches_v": caches_v,
    }
    return x


def _check(x, lens, window, R, scale, max_seq_len, temp_n0=0, label=""):
    B, Hq, _ = x["q"].shape
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    o = ops.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["table"], x["lens"], x["r"], x["w"], window, R,
                              max_seq_len, scale, lse=lse, temp_n0=temp_n0)
    torch.cuda.synchronize()
    for b, n in enumerate(lens):
        o_ref, lse_ref = O.attn_decode(x["q"][b:b + 1].cpu(), x["caches_k"][b][None].cpu(),
                                       x["caches_v"][b][None].cpu(), x["r"][b:b + 1].cpu(), x["w"].cpu(), window, R,
                                       scale, temp_n0=temp_n0)
        assert_bf16_close(o[b:b + 1], o_ref, lse[b:b + 1], lse_ref, "%s seq %d (n=%d)" % (label, b, n))
    return o, lse


@pytest.mark.parametrize("lens,Hq,Hkv,window,R,page_size,temp_n0", [
    ([1, 31, 32, 100], 8, 2, 0, 64, 32, 0),              # one row, chunk edge, several pages
    ([1000, 2049, 777], 8, 1, 512, 512, 256, 0),         # windowed: chunks aligned below the window start
    ([5000, 64], 32, 4, 0, 1024, 64, 1000),              # global-layer heads, temperature past 1000 keys
    ([333, 4096, 1, 2500], 16, 4, 0, 300, 128, 0),
    ([700, 129], 12, 3, 100, 50, 96, 0),                 # page size not a power of two
])
def test_paged_decode_parity(lens, Hq, Hkv, window, R, page_size, temp_n0):
    x = _paged_inputs(lens, Hq, Hkv, R, page_size, seed=sum(lens) + page_size)
    _check(x, lens, window, R, 1.0 / math.sqrt(128), max(lens), temp_n0, "paged %s" % ((lens, window, R),))


def test_paged_decode_short_sequences_under_a_long_bound():
    """max_seq_len plans the splits; sequences far shorter leave most splits empty."""
    lens = [40, 3, 130]
    x = _paged_inputs(lens, 8, 2, 64, 32, seed=5, max_seq_len=200000)
    _check(x, lens, 0, 64, 0.0884, max_seq_len=200000, label="short under long bound")


def test_paged_matches_contiguous_decode_bitwise():
    """In-order pages holding a whole cache give the contiguous entry point's bits."""
    B, N, Hq, Hkv, R, d = 2, 3000, 8, 2, 512, 128
    k = synth.normal((B, N, Hkv, d), 77, "k", dtype=torch.bfloat16, device="cuda")
    v = synth.normal((B, N, Hkv, d), 77, "v", dtype=torch.bfloat16, device="cuda")
    q = synth.normal((B, Hq, d), 77, "q", dtype=torch.bfloat16, device="cuda")
    r = synth.normal((B, Hq), 77, "r", device="cuda")
    w = synth.normal((Hq, R), 77, "w", std=0.5, device="cuda")
    page = 3008   # 94 chunks of 32 rows: one page per sequence
    pool_k = torch.zeros(B, page, Hkv, d, dtype=torch.bfloat16, device="cuda")
    pool_v = torch.zeros_like(pool_k)
    pool_k[:, :N] = k
    pool_v[:, :N] = v
    table = torch.arange(B, dtype=torch.int32, device="cuda").reshape(B, 1)
    lens = torch.full((B,), N, dtype=torch.int32, device="cuda")
    o1 = ops.attn_decode(q, k, v, r, w, 0, R, 0.0884)
    o2 = ops.attn_decode_paged(q, pool_k, pool_v, table, lens, r, w, 0, R, N, 0.0884)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_paged_decode_reports_a_length_past_the_bound():
    lens = [100, 50]
    x = _paged_inputs(lens, 8, 2, 64, 32, seed=9)
    bad = torch.tensor([100, 500], dtype=torch.int32, device="cuda")   # 500 > max_seq_len = 100
    o = ops.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["table"], bad, x["r"], x["w"], 0, 64, 100,
                              0.0884)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.RELBIAS_STATUS_BAD_LENGTH
    assert torch.isfinite(o[0].float()).all()   # the valid sequence is unaffected by the clamped one


def test_paged_decode_workload_sampled():
    """The 8 x 1,048,576-row paged decode workload (256-row pages, shuffled pool), in
    the launch configuration the benchmark times, checked on sampled (sequence,
    key/value head) groups against the oracle on that group's logical cache."""
    from attention_learned_relative_b200.workloads import WORKLOADS, logical_cache, make_inputs
    wl = WORKLOADS["global_decode_paged_bf16"]
    x = make_inputs(wl, device="cuda")
    B, Hq, d = x["q"].shape
    N = wl.T
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    o = ops.attn_decode_paged(x["q"], x["k_pages"], x["v_pages"], x["table"], x["lens"], x["r"], x["w"],
                              wl.window, wl.R, N, wl.scale, lse=lse)
    torch.cuda.synchronize()
    G = wl.group
    for (b, g) in [(1, 2), (6, 0)]:
        heads = list(range(g * G, (g + 1) * G))
        k_sl, v_sl = logical_cache(x, b, g)
        req = np.array([(0, hl, N - 1) for hl in range(G)], dtype=np.int64)
        o_ref, lse_ref = O.attn_rows(x["q"][b, heads].float().cpu(), x["r"][b, heads].cpu().reshape(G, 1),
                                     x["w"][heads].cpu().reshape(G, 1, wl.R), k_sl[None].cpu(), v_sl[None].cpu(),
                                     req, G, wl.window, wl.R, wl.scale)
        assert_bf16_close(o[b, heads], o_ref, lse[b, heads], lse_ref, "paged decode workload (b=%d, g=%d)" % (b, g))
