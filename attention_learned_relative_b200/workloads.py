"""The synthetic workloads the library is checked and timed on.

Shapes follow the pages' two layer types: local layers attend a 512-key sliding
window with a 512-distance bias, global layers are fully causal with the bias over
the last 1024 distances and content-only attention beyond ("Learned
Relative-Position Bias", codewithdark concepts page, "Hybrid Attention
Interaction"; banandre.com deep dive, "No RoPE? No Problem?").  32 query heads on 4
key/value heads (GQA), head dim 128, and a 1,048,576-token context for decode
(archdiff.com model card, "Context").  Values: Q, K, V ~ N(0,1) rounded to bf16,
r ~ N(0,1) and w ~ N(0, 0.5^2) in fp32, all from `synth` with a per-workload seed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int            # tokens per sequence (prefill) or cache rows n_ctx (decode)
    Hq: int
    Hkv: int
    d: int
    window: int       # <= 0: full causal
    R: int
    seed: int
    dtype: str        # "fp32" or "bf16"
    decode: bool = False
    qk_std: float = 1.0   # Q and K are drawn as N(0, qk_std^2)
    page_size: int = 0    # decode only: > 0 stores the cache as shuffled pages of this many rows
    bank_C: int = 0       # > 0: shared-bank bias with this many functions (rs, proj inputs)
    backward: bool = False  # prefill only: the step is the backward pass (dout input, gradients out)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def attended_pairs(self) -> int:
        """Number of (query, key) pairs inside the causal mask and window, per (b, h)."""
        if self.decode:
            return self.T if self.window <= 0 else min(self.T, self.window)
        T, W = self.T, self.window
        if W <= 0 or W >= T:
            return T * (T + 1) // 2
        return W * (W + 1) // 2 + (T - W) * W

    def masked_flops(self) -> int:
        """2 flops per multiply-add of QK^T and PV over attended pairs only.  For a
        backward workload: the five products of the backward pass (QK^T recomputed,
        dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q), 2.5 times the forward."""
        per_pair = 10 * self.d if self.backward else 4 * self.d
        return per_pair * self.attended_pairs() * self.B * self.Hq

    def kv_bytes(self) -> int:
        """Bytes of K and V a decode step must stream (the attended cache rows)."""
        esz = 2 if self.dtype == "bf16" else 4
        return 2 * self.B * self.Hkv * self.attended_pairs() * self.d * esz

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_local_fp32", B=1, T=256, Hq=4, Hkv=1, d=64, window=64, R=64,
                 seed=0, dtype="fp32"),
        Workload("local_prefill_bf16", B=2, T=8192, Hq=32, Hkv=4, d=128, window=512, R=512,
                 seed=1, dtype="bf16"),
        Workload("global_prefill_bf16", B=1, T=32768, Hq=32, Hkv=4, d=128, window=0, R=1024,
                 seed=2, dtype="bf16"),
        Workload("global_long_prefill_bf16", B=1, T=131072, Hq=32, Hkv=4, d=128, window=0,
                 R=1024, seed=3, dtype="bf16", qk_std=0.5),
        Workload("global_decode_bf16", B=8, T=1048576, Hq=32, Hkv=4, d=128, window=0, R=1024,
                 seed=4, dtype="bf16", decode=True),
        # The same decode step against a paged cache: 256-row pages in a pool whose
        # block table is a seeded random permutation (scattered physical pages).
        Workload("global_decode_paged_bf16", B=8, T=1048576, Hq=32, Hkv=4, d=128, window=0,
                 R=1024, seed=4, dtype="bf16", decode=True, page_size=256),
        # The same decode step with the essay's shared-bank bias: 16 functions of
        # distance shared by all heads, 16 coefficients per (token, head).
        Workload("global_decode_bank_bf16", B=8, T=1048576, Hq=32, Hkv=4, d=128, window=0,
                 R=1024, seed=4, dtype="bf16", decode=True, bank_C=16),
        # The local-layer prefill with the essay's shared bank: 16 functions of distance
        # shared by all heads, 16 coefficients per (token, head).
        Workload("local_prefill_bank_bf16", B=2, T=8192, Hq=32, Hkv=4, d=128, window=512, R=512,
                 seed=1, dtype="bf16", bank_C=16),
        # The backward pass of the local-layer prefill (the pages train the model).
        Workload("local_backward_bf16", B=2, T=8192, Hq=32, Hkv=4, d=128, window=512, R=512,
                 seed=1, dtype="bf16", backward=True),
        # The same backward with the shared-bank bias (16 functions shared by all heads).
        Workload("local_backward_bank_bf16", B=2, T=8192, Hq=32, Hkv=4, d=128, window=512, R=512,
                 seed=1, dtype="bf16", backward=True, bank_C=16),
    ]
}


def make_inputs(wl: Workload, device="cpu", T: int | None = None, B: int | None = None, kv=None):
    """Inputs of a workload (optionally with fewer tokens or sequences), on `device`.

    Prefill: q [B,T,Hq,d], k/v [B,T,Hkv,d] (wl dtype), r [B,T,Hq] fp32, w [Hq,R] fp32.
    Decode:  q [B,Hq,d], k/v [B,T,Hkv,d] (the cache), r [B,Hq] fp32, w [Hq,R] fp32.
    Paged decode (page_size > 0) adds k_pages/v_pages [B*T/page_size, page_size, Hkv, d]
    (the same storage as k/v, read as a page pool), table [B, T/page_size] int32 (a
    seeded permutation of the pool: sequence b's logical block j is page table[b, j])
    and lens [B] int32.  The logical cache of sequence b is then k_pages[table[b]],
    not k[b]; logical_cache() returns it.
    `kv`, if given, is a (k, v) pair drawn earlier for the same seed and shape, used
    instead of drawing the same values again.
    """
    T = wl.T if T is None else T
    B = wl.B if B is None else B
    dt = wl.torch_dtype()
    s = wl.seed
    if wl.decode:
        q = synth.normal((B, wl.Hq, wl.d), s, "q", dtype=dt, device=device)
        r = synth.normal((B, wl.Hq), s, "r", device=device)
    else:
        q = synth.normal((B, T, wl.Hq, wl.d), s, "q", std=wl.qk_std, dtype=dt, device=device)
        r = synth.normal((B, T, wl.Hq), s, "r", device=device)
    if kv is not None:
        k, v = kv
        if tuple(k.shape) != (B, T, wl.Hkv, wl.d) or k.dtype != dt or v.shape != k.shape:
            raise ValueError("kv does not match the workload's cache shape")
    else:
        k = synth.normal((B, T, wl.Hkv, wl.d), s, "k", std=wl.qk_std, dtype=dt, device=device)
        v = synth.normal((B, T, wl.Hkv, wl.d), s, "v", dtype=dt, device=device)
    w = synth.normal((wl.Hq, wl.R), s, "w", std=0.5, device=device)
    x = {"q": q, "k": k, "v": v, "r": r, "w": w}
    if wl.backward:
        x["dout"] = synth.normal((B, T, wl.Hq, wl.d), s, "bank", dtype=dt, device=device)
    if wl.bank_C > 0:
        # Shared bank: rs ~ N(0, 1/C) coefficients and proj ~ N(0, 0.5^2) functions, so a
        # curve value sum_c rs[c] proj[c, dist] has the spread of r * w (std 0.5).
        C = wl.bank_C
        shape = (B, wl.Hq, C) if wl.decode else (B, T, wl.Hq, C)
        x["rs"] = synth.normal(shape, s, "rs", std=1.0 / math.sqrt(C), device=device)
        x["proj"] = synth.normal((1, C, wl.R), s, "proj", std=0.5, device=device)
    if wl.decode and wl.page_size > 0:
        if T % wl.page_size != 0:
            raise ValueError("paged workload needs T (%d) divisible by page_size (%d)" % (T, wl.page_size))
        npb = T // wl.page_size
        x["k_pages"] = k.view(B * npb, wl.page_size, wl.Hkv, wl.d)
        x["v_pages"] = v.view(B * npb, wl.page_size, wl.Hkv, wl.d)
        g = torch.Generator().manual_seed(s + 77)
        x["table"] = torch.randperm(B * npb, generator=g).to(torch.int32).reshape(B, npb).to(device)
        x["lens"] = torch.full((B,), T, dtype=torch.int32, device=device)
    return x


def logical_cache(x, b: int, kv: int | None = None):
    """(K, V) of sequence b in logical row order, [T, Hkv, d] (or [T, 1, d] for one
    key/value head), gathered through the block table for a paged workload."""
    if "table" not in x:
        ks, vs = x["k"][b], x["v"][b]
    else:
        pages = x["table"][b].long()
        ks = x["k_pages"][pages].flatten(0, 1)
        vs = x["v_pages"][pages].flatten(0, 1)
    if kv is not None:
        ks, vs = ks[:, kv:kv + 1], vs[:, kv:kv + 1]
    return ks, vs
