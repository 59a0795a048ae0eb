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
        """2 flops per multiply-add of QK^T and PV over attended pairs only."""
        return 4 * self.d * self.attended_pairs() * self.B * self.Hq

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
    ]
}


def make_inputs(wl: Workload, device="cpu", T: int | None = None, B: int | None = None):
    """Inputs of a workload (optionally with fewer tokens or sequences), on `device`.

    Prefill: q [B,T,Hq,d], k/v [B,T,Hkv,d] (wl dtype), r [B,T,Hq] fp32, w [Hq,R] fp32.
    Decode:  q [B,Hq,d], k/v [B,T,Hkv,d] (the cache), r [B,Hq] fp32, w [Hq,R] fp32.
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
    k = synth.normal((B, T, wl.Hkv, wl.d), s, "k", std=wl.qk_std, dtype=dt, device=device)
    v = synth.normal((B, T, wl.Hkv, wl.d), s, "v", dtype=dt, device=device)
    w = synth.normal((wl.Hq, wl.R), s, "w", std=0.5, device=device)
    return {"q": q, "k": k, "v": v, "r": r, "w": w}
