"""GPU parity of chunked prefill against a paged, variable-length cache
(relbias_attn_fwd_chunk_paged): every sequence has its own chunk offset and length,
its cache rows live in shuffled pages of a pool, and unused pages and rows past each
sequence's end hold NaN (stale rows of a serving cache), so a kernel that let them
into a product would fail.  The oracle computes the same rows of each whole sequence.
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
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out or read a bad length"


def _case(offs, lens, T, Hq, Hkv, d, R, page, seed, spare_pages=3):
    """Sequences of length offs[b] + lens[b] (their whole rows drawn), written into a
    shuffled page pool with NaN everywhere else; q/r hold each chunk's rows (rows past
    lens[b] are NaN too)."""
    B = len(offs)
    dev = "cuda"
    L = max(o + n for o, n in zip(offs, lens))
    full = {
        "q": synth.normal((B, L, Hq, d), seed, "q", dtype=torch.bfloat16, device=dev),
        "k": synth.normal((B, L, Hkv, d), seed, "k", dtype=torch.bfloat16, device=dev),
        "v": synth.normal((B, L, Hkv, d), seed, "v", dtype=torch.bfloat16, device=dev),
        "r": synth.normal((B, L, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
    }
    max_pages = (L + page - 1) // page
    num_pages = B * max_pages + spare_pages
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    kp = torch.full((num_pages, page, Hkv, d), float("nan"), dtype=torch.bfloat16, device=dev)
    vp = torch.full_like(kp, float("nan"))
    nxt = 0
    for b in range(B):
        n = offs[b] + lens[b]
        for blk in range((n + page - 1) // page):
            pg = int(perm[nxt])
            nxt += 1
            table[b, blk] = pg
            rows = min(page, n - blk * page)
            kp[pg, :rows] = full["k"][b, blk * page:blk * page + rows]
            vp[pg, :rows] = full["v"][b, blk * page:blk * page + rows]
    q = torch.full((B, T, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    r = torch.full((B, T, Hq), float("nan"), dtype=torch.float32, device=dev)
    for b in range(B):
        q[b, :lens[b]] = full["q"][b, offs[b]:offs[b] + lens[b]]
        r[b, :lens[b]] = full["r"][b, offs[b]:offs[b] + lens[b]]
    return full, q, r, kp, vp, table.to(dev), torch.tensor(offs, dtype=torch.int32, device=dev), \
        torch.tensor(lens, dtype=torch.int32, device=dev)


CASES = [
    # offs,             lens,           T,   Hq, Hkv, d,   window, R,   page, temp_n0
    ([0, 300, 1000],    [200, 128, 50], 200, 8, 2, 128, 0, 256, 128, 0),
    ([129, 0],          [257, 64],      257, 8, 2, 128, 512, 512, 64, 0),     # local layer
    ([700, 64, 5],      [64, 1, 100],   100, 6, 2, 64, 128, 100, 192, 0),     # d 64, group 3
    ([2000, 33],        [100, 300],     300, 4, 1, 128, 0, 1024, 128, 600),   # global, temperature
    ([50, 500],         [0, 40],        40, 8, 2, 128, 0, 64, 64, 0),         # an empty chunk
]


@pytest.mark.parametrize("offs,lens,T,Hq,Hkv,d,window,R,page,temp_n0", CASES)
def test_chunk_paged_parity(offs, lens, T, Hq, Hkv, d, window, R, page, temp_n0):
    full, q, r, kp, vp, table, qo, ql = _case(offs, lens, T, Hq, Hkv, d, R, page, seed=sum(offs) + T + d)
    scale = 1.0 / math.sqrt(d)
    sentinel = -7.0
    o = torch.full_like(q, sentinel)
    lse = torch.full((len(offs), Hq, T), sentinel, dtype=torch.float32, device="cuda")
    ops.attn_fwd_chunk_paged(q, kp, vp, table, qo, ql, r, full["w"], window, R, scale, out=o, lse=lse,
                             temp_n0=temp_n0)
    torch.cuda.synchronize()
    for b, (off, n) in enumerate(zip(offs, lens)):
        # rows past the chunk's length are not written
        assert bool((o[b, n:] == sentinel).all()) and bool((lse[b, :, n:] == sentinel).all())
        if n == 0:
            continue
        rows = np.array([(0, h, off + i) for h in range(Hq) for i in range(n)], dtype=np.int64)
        L = off + n
        o_ref, lse_ref = O.attn_prefill(full["q"][b:b + 1, :L].cpu(), full["k"][b:b + 1, :L].cpu(),
                                        full["v"][b:b + 1, :L].cpu(), full["r"][b:b + 1, :L].cpu(), full["w"].cpu(),
                                        window, R, scale, rows=rows, temp_n0=temp_n0)
        got = o[b, :n].permute(1, 0, 2).reshape(-1, d)       # (h, i) order, as `rows`
        got_lse = lse[b, :, :n].reshape(-1)
        assert_bf16_close(got, o_ref, got_lse, lse_ref, "paged chunk b=%d %s" % (b, (offs, lens, window, R, page)))


def test_chunk_paged_matches_contiguous_chunk():
    """One sequence, pages in order: the paged kernel and the contiguous chunk kernel
    compute the same rows (the same tile stream and arithmetic)."""
    off, n, Hq, Hkv, d, R, page = 300, 200, 8, 2, 128, 256, 128
    full, q, r, kp, vp, table, qo, ql = _case([off], [n], n, Hq, Hkv, d, R, page, seed=5, spare_pages=0)
    o1 = ops.attn_fwd_chunk_paged(q, kp, vp, table, qo, ql, r, full["w"], 0, R, 0.09)
    o2 = ops.attn_fwd_chunk(q, full["k"][:, :off + n].contiguous(), full["v"][:, :off + n].contiguous(), r,
                            full["w"], off, 0, R, 0.09)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2


def test_chunk_paged_bad_length_is_reported():
    """An offset + length past the table's capacity is clamped and reported, not read."""
    full, q, r, kp, vp, table, qo, ql = _case([10], [50], 50, 4, 2, 128, 32, 64, seed=8)
    bad = torch.tensor([table.shape[1] * 64], dtype=torch.int32, device="cuda")   # offset at capacity
    ops.attn_fwd_chunk_paged(q, kp, vp, table, bad, ql, r, full["w"], 0, 32, 0.1)
    assert ops.device_status(reset=True) & ops.RELBIAS_STATUS_BAD_LENGTH
