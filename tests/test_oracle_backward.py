"""Pins of the oracle's backward pass (oracle_attn_bwd) to something other than itself:
central finite differences of the forward oracle, which is pinned on its own
(test_oracle_pins.py).  The loss is L = sum(dout * O); every input is perturbed by
+-eps with eps a power of two, so the perturbed float32 inputs are exact, and two
step sizes are combined by Richardson extrapolation (error O(eps^4)).
"""
import numpy as np
import pytest
import torch

from attention_learned_relative_b200 import synth
from oracle import oracle as O


def _loss(x, dout, window, R, scale, temp_n0):
    o, _ = O.attn_prefill(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, scale, temp_n0=temp_n0)
    return float((o * dout.astype(np.float64)).sum())


def _fd(x, dout, name, idx, window, R, scale, temp_n0):
    def at(eps):
        vals = []
        for sgn in (+1, -1):
            y = {k: t.copy() for k, t in x.items()}
            y[name][idx] += np.float32(sgn * eps)
            vals.append(_loss(y, dout, window, R, scale, temp_n0))
        return (vals[0] - vals[1]) / (2 * eps)
    e = 2.0 ** -7
    return (4 * at(e / 2) - at(e)) / 3


CASES = [
    # B, T,  Hq, Hkv, d,  window, R,  C,  proj_heads, temp_n0
    (1, 13, 2, 1, 8, 0, 9, 1, 2, 0),      # rank-1 per head, causal
    (2, 11, 4, 2, 8, 5, 7, 1, 4, 0),      # window, GQA
    (1, 12, 2, 2, 8, 0, 12, 3, 1, 0),     # shared bank of 3 functions
    (1, 14, 2, 1, 8, 0, 6, 1, 2, 4),      # temperature: tau > 1 for rows seeing > 4 keys
    (1, 10, 2, 1, 8, 4, 8, 2, 2, 0),      # a bank of 2 functions per head, window
]


@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R,C,proj_heads,temp_n0", CASES)
def test_backward_matches_finite_differences(B, T, Hq, Hkv, d, window, R, C, proj_heads, temp_n0):
    seed = 100 + T + C
    x = {
        "q": synth.normal((B, T, Hq, d), seed, "q").numpy(),
        "k": synth.normal((B, T, Hkv, d), seed, "k").numpy(),
        "v": synth.normal((B, T, Hkv, d), seed, "v").numpy(),
        "r": synth.normal((B, T, Hq) if C == 1 else (B, T, Hq, C), seed, "r").numpy(),
        "w": synth.normal((Hq, R) if (C == 1 and proj_heads == Hq) else (proj_heads, C, R), seed, "w",
                          std=0.5).numpy(),
    }
    dout = synth.normal((B, T, Hq, d), seed, "bank").numpy()
    scale = 0.4
    rng = np.random.default_rng(seed)
    names = {"q": "dq", "k": "dk", "v": "dv", "r": "dr", "w": "dw"}
    picks = []
    for name in names:
        for _ in range(4):
            idx = tuple(int(rng.integers(0, s)) for s in x[name].shape)
            # Snap the entry to a multiple of 2^-10, so that it plus or minus 2^-7 or 2^-8
            # is exact in float32 (no rounding at a binade boundary).
            x[name][idx] = np.float32(np.round(float(x[name][idx]) * 1024.0) / 1024.0)
            picks.append((name, idx))
    g = O.attn_backward(x["q"], x["k"], x["v"], x["r"], x["w"], dout, window, R, scale, temp_n0=temp_n0)
    for name, idx in picks:
        fd = _fd(x, dout, name, idx, window, R, scale, temp_n0)
        an = g[names[name]][idx]
        assert abs(fd - an) <= 1e-8 + 1e-7 * abs(an), (name, idx, fd, an)


def test_backward_of_zero_table_has_zero_feature_gradient():
    """With w = 0 the bias vanishes for every r, so dL/dr = 0 exactly; dL/dw does not vanish."""
    B, T, Hq, Hkv, d, R = 1, 10, 2, 1, 8, 6
    q = synth.normal((B, T, Hq, d), 5, "q").numpy()
    k = synth.normal((B, T, Hkv, d), 5, "k").numpy()
    v = synth.normal((B, T, Hkv, d), 5, "v").numpy()
    r = synth.normal((B, T, Hq), 5, "r").numpy()
    w = np.zeros((Hq, R), dtype=np.float32)
    dout = synth.normal((B, T, Hq, d), 5, "bank").numpy()
    g = O.attn_backward(q, k, v, r, w, dout, 0, R, 0.3)
    assert np.all(g["dr"] == 0.0)
    assert np.abs(g["dw"]).max() > 1e-3


def test_value_gradient_is_attention_transpose_times_dout():
    """dV = P^T dO exactly, with P rebuilt from the brute-force bias matrix and a plain
    fp64 softmax (a second, independent route to the same numbers)."""
    T, H, d, R = 9, 1, 4, 5
    q = synth.normal((1, T, H, d), 8, "q").double()
    k = synth.normal((1, T, H, d), 8, "k").double()
    v = synth.normal((1, T, H, d), 8, "v").double()
    r = synth.normal((1, T, H), 8, "r").double()
    w = synth.normal((H, R), 8, "w", std=0.5).double()
    dout = synth.normal((1, T, H, d), 8, "bank").double()
    bias = O.bias_matrix(r[0].reshape(T, H, 1).numpy(), w.reshape(H, 1, R).numpy(), np.arange(T), R)[0]
    logits = 0.5 * (q[0, :, 0] @ k[0, :, 0].T).numpy() + bias
    logits[np.triu_indices(T, 1)] = -np.inf
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    dv_ref = p.T @ dout[0, :, 0].numpy()
    g = O.attn_backward(q.float(), k.float(), v.float(), r.float(), w.float(), dout.float(), 0, R, 0.5)
    np.testing.assert_allclose(g["dv"][0, :, 0], dv_ref, rtol=1e-6, atol=1e-6)
