"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics, not by the
oracle's own code.

* hand-worked cases (tests/golden/hand_worked.json) with exact rational answers;
* w = 0 reduces to plain causal / windowed attention: torch's
  scaled_dot_product_attention in fp64 on the CPU (the pages' NoPE layers);
* r = 1, w[h, d] = -m_h * d reduces to ALiBi (the linear penalty the concepts
  page lists under "Variants / Extensions"), again through the library routine;
* Q = 0 with one-hot values reads the attention probabilities out directly; their
  log-ratios must equal r_i * (w[i-j] - w[0]) inside R and -r_i * w[0] beyond;
* constant V, K = 0, a bias that is constant per row (softmax shift invariance);
* local-layer locality and the global-layer positionless far field (tokens beyond
  the window do not matter; keys beyond R with equal K get equal weight).

Each of these fails for a plausible slip in the oracle: a dropped bias or scale, a
j-i for i-j, r_j for r_i, another head's table, an off-by-one at R or at the
window edge, a transposed operand, or a wrong LSE.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _num(s):
    """Parse the fixture's exact expressions: '6/5', 'ln7', 'ln3/2', '0'."""
    if isinstance(s, (int, float)):
        return float(s)
    s = s.strip()
    if s.startswith("ln"):
        rest = s[2:]
        if "/" in rest:
            a, b = rest.split("/")
            return math.log(float(a)) / float(b)
        return math.log(float(rest))
    return float(Fraction(s))


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _sdpa(q, k, v, scale, window, extra_bias=None):
    """torch SDPA in fp64 with the causal (and window) mask; q [B,T,Hq,d], k/v [B,T,Hkv,d].
    GQA: query head h reads key/value head h // (Hq/Hkv)."""
    B, T, Hq, d = q.shape
    G = Hq // k.shape[2]
    qh = q.permute(0, 2, 1, 3)
    kh = k.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vh = v.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = (j <= i)
    if window > 0:
        allowed = allowed & (i - j < window)
    mask = torch.zeros(T, T, dtype=torch.float64).masked_fill(~allowed, float("-inf"))
    mask = mask.expand(B, Hq, T, T)
    if extra_bias is not None:
        mask = mask + extra_bias
    o = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3)


def _attended(i, window):
    lo = 0 if window <= 0 else max(0, i - window + 1)
    return list(range(lo, i + 1))


# ---------------------------------------------------------------------------


def test_golden_hand_worked(oracle):
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        T, d, R = c["T"], c["d"], c["R"]
        q = np.array(c["q"], dtype=np.float32).reshape(1, T, 1, d)
        k = np.array(c["k"], dtype=np.float32).reshape(1, T, 1, d)
        v = np.array(c["v"], dtype=np.float32).reshape(1, T, 1, d)
        r = np.array(c["r"], dtype=np.float32).reshape(1, T, 1)
        w = np.array([_num(x) for x in c["w"]], dtype=np.float32).reshape(1, R)
        scale = _num(c["scale"])
        o, lse = oracle.attn_prefill(q, k, v, r, w, c["window"], R, scale)
        want_o = np.array([[_num(x) for x in row] for row in c["expect_o"]])
        want_lse = np.array([_num(x) for x in c["expect_lse"]])
        # w and scale pass through float32, so allow for its rounding of ln values.
        np.testing.assert_allclose(o[0, :, 0, :], want_o, rtol=1e-6, atol=1e-7, err_msg=c["name"])
        np.testing.assert_allclose(lse[0, 0, :], want_lse, rtol=1e-6, atol=1e-7, err_msg=c["name"])


@pytest.mark.parametrize("window", [0, 1, 5, 16])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2), (8, 1)])
def test_nope_reduces_to_sdpa(oracle, window, Hq, Hkv):
    """w = 0: plain causal (or sliding-window) attention, checked against torch SDPA."""
    B, T, d, R = 2, 37, 16, 8
    q, k, v = _rand((B, T, Hq, d), 1), _rand((B, T, Hkv, d), 2), _rand((B, T, Hkv, d), 3)
    r = _rand((B, T, Hq), 4)
    w = torch.zeros(Hq, R, dtype=torch.float64)
    q, k, v = (x.float().double() for x in (q, k, v))  # values exact in float32
    scale = 0.3
    o, _ = oracle.attn_prefill(q, k, v, r, w, window, R, scale)
    ref = _sdpa(q, k, v, scale, window).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_r_zero_also_reduces_to_sdpa(oracle):
    B, T, Hq, Hkv, d, R = 1, 29, 4, 4, 8, 64
    q, k, v = (_rand(s, i).float().double() for i, s in enumerate([(B, T, Hq, d), (B, T, Hkv, d), (B, T, Hkv, d)]))
    w = _rand((Hq, R), 9).float()
    r = torch.zeros(B, T, Hq)
    o, _ = oracle.attn_prefill(q, k, v, r, w, 0, R, 0.25)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.25, 0).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [0, 7])
def test_alibi_reduction(oracle, window):
    """r = 1 and w[h, d] = -m_h * d with R beyond every distance is ALiBi."""
    B, T, Hq, Hkv, d = 1, 33, 4, 2, 8
    R = T + 3
    slopes = torch.tensor([2.0 ** (-(h + 1)) for h in range(Hq)], dtype=torch.float64)
    q, k, v = (_rand(s, 10 + i).float().double() for i, s in enumerate([(B, T, Hq, d), (B, T, Hkv, d), (B, T, Hkv, d)]))
    r = torch.ones(B, T, Hq)
    w = (-slopes[:, None] * torch.arange(R, dtype=torch.float64)[None, :]).float()
    o, _ = oracle.attn_prefill(q, k, v, r, w, window, R, 0.5)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    alibi = (-slopes[:, None, None] * (i - j).clamp(min=0).double()[None]).float().double()
    ref = _sdpa(q, k, v, 0.5, window, extra_bias=alibi[None]).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-7)


@pytest.mark.parametrize("window,R", [(0, 5), (6, 4), (9, 9), (0, 1)])
def test_probabilities_closed_form(oracle, window, R):
    """Q = 0 and V = identity: O[i, j] is the weight of key j.  Its log-ratio to the
    self weight must be r_i*(w[h,i-j] - w[h,0]) inside R and -r_i*w[h,0] beyond."""
    T, Hq = 16, 3
    d = T
    q = torch.zeros(1, T, Hq, d)
    k = _rand((1, T, 1, d), 20).float()
    v = torch.eye(T).reshape(1, T, 1, d)
    r = _rand((1, T, Hq), 21).float()
    w = _rand((Hq, R), 22).float()
    o, lse = oracle.attn_prefill(q, k, v, r, w, window, R, 0.7)
    r64, w64 = r.double().numpy(), w.double().numpy()
    for h in range(Hq):
        for i in range(T):
            p = o[0, i, h, :]
            att = _attended(i, window)
            outside = [j for j in range(T) if j not in att]
            assert np.all(p[outside] == 0.0)
            assert abs(p.sum() - 1.0) < 1e-13
            for j in att:
                dist = i - j
                expect = r64[0, i, h] * ((w64[h, dist] if dist < R else 0.0) - w64[h, 0])
                assert abs(math.log(p[j]) - math.log(p[i]) - expect) < 1e-12
            # LSE consistent with the self weight: p_ii = exp(r_i*w[0] - LSE_i)
            assert abs(lse[0, h, i] - (r64[0, i, h] * w64[h, 0] - math.log(p[i]))) < 1e-12


def test_probabilities_match_listing_bias_matrix(oracle):
    """The same read-out against the (H, T, T) bias built entry by entry, for a
    rank-4 bank shared by all heads (the essay's 16-function bank, smaller)."""
    T, H, C, R = 12, 2, 4, 7
    d = T
    rs = _rand((T, H, C), 30).float()
    bank = _rand((C, R), 31).float()
    q = torch.zeros(1, T, H, d)
    k = _rand((1, T, 1, d), 32).float()
    v = torch.eye(T).reshape(1, T, 1, d)
    o, _ = oracle.attn_prefill(q, k, v, rs.reshape(1, T, H, C), bank, 0, R, 1.0)
    bias = oracle.bias_matrix(rs.double().numpy(), bank.double().numpy(), np.arange(T), R)
    for h in range(H):
        for i in range(T):
            for j in range(i + 1):
                got = math.log(o[0, i, h, j]) - math.log(o[0, i, h, i])
                assert abs(got - (bias[h, i, j] - bias[h, i, i])) < 1e-11


def test_bank_alibi_reduction(oracle):
    """A shared bank whose first function is -distance and whose coefficients are the
    head slopes (all other coefficients 0) is again ALiBi."""
    B, T, Hq, d, C = 1, 20, 2, 4, 3
    R = T
    slopes = [0.5, 0.125]
    bank = _rand((C, R), 40).float()
    bank[0] = -torch.arange(R, dtype=torch.float32)
    rs = torch.zeros(B, T, Hq, C)
    for h in range(Hq):
        rs[:, :, h, 0] = slopes[h]
    q, k, v = (_rand(s, 41 + i).float().double() for i, s in enumerate([(B, T, Hq, d), (B, T, 1, d), (B, T, 1, d)]))
    o, _ = oracle.attn_prefill(q, k, v, rs, bank, 0, R, 0.5)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    sl = torch.tensor(slopes, dtype=torch.float64)
    alibi = -sl[:, None, None] * (i - j).clamp(min=0).double()[None]
    ref = _sdpa(q, k, v, 0.5, 0, extra_bias=alibi[None]).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-7)


def test_constant_values(oracle):
    B, T, Hq, Hkv, d, R = 2, 21, 4, 2, 8, 6
    q, k = _rand((B, T, Hq, d), 50).float(), _rand((B, T, Hkv, d), 51).float()
    c = torch.linspace(-2, 3, d)
    v = c.expand(B, T, Hkv, d).contiguous()
    o, _ = oracle.attn_prefill(q, k, v, _rand((B, T, Hq), 52).float(), _rand((Hq, R), 53).float(), 4, R, 0.4)
    np.testing.assert_allclose(o, np.broadcast_to(c.double().numpy(), o.shape), rtol=0, atol=1e-14)


@pytest.mark.parametrize("window", [0, 6])
def test_zero_keys_no_bias_gives_mean(oracle, window):
    B, T, Hq, d, R = 1, 19, 2, 5, 4
    q = _rand((B, T, Hq, d), 60).float()
    k = torch.zeros(B, T, 1, d)
    v = _rand((B, T, 1, d), 61).float()
    o, lse = oracle.attn_prefill(q, k, v, _rand((B, T, Hq), 62).float(), torch.zeros(Hq, R), window, R, 1.0)
    v64 = v.double().numpy()
    for i in range(T):
        att = _attended(i, window)
        np.testing.assert_allclose(o[0, i, 0], v64[0, att, 0].mean(axis=0), rtol=0, atol=1e-14)
        assert abs(lse[0, 1, i] - math.log(len(att))) < 1e-14


def test_constant_bias_lse(oracle):
    """Q = 0, r = 1, w[h] = c_h and window <= R: every logit is c_h, so
    LSE_i = c_h + log|A_i| and O_i is the mean of V over A_i."""
    T, Hq, d, W, R = 25, 3, 4, 5, 8
    cs = [0.75, -1.5, 2.0]
    w = torch.tensor([[c] * R for c in cs])
    v = _rand((1, T, 1, d), 70).float()
    o, lse = oracle.attn_prefill(torch.zeros(1, T, Hq, d), _rand((1, T, 1, d), 71).float(), v,
                                 torch.ones(1, T, Hq), w, W, R, 0.9)
    for h in range(Hq):
        for i in range(T):
            att = _attended(i, W)
            assert abs(lse[0, h, i] - (cs[h] + math.log(len(att)))) < 1e-12
            np.testing.assert_allclose(o[0, i, h], v.double().numpy()[0, att, 0].mean(0), atol=1e-14)


def test_bias_shift_invariance(oracle):
    """Adding a constant to w shifts row i's logits by r_i * c uniformly when the whole
    window lies inside R; the output must not move.  (Scaling by r_j instead of r_i
    would shift each key differently and fail.)"""
    B, T, Hq, Hkv, d, W, R = 1, 30, 2, 1, 8, 6, 6
    q, k, v = (_rand(s, 80 + i).float() for i, s in enumerate([(B, T, Hq, d), (B, T, Hkv, d), (B, T, Hkv, d)]))
    r = _rand((B, T, Hq), 83).float()
    w = _rand((Hq, R), 84).bfloat16().float()   # few mantissa bits: w + 1.25 is exact in fp32
    o1, _ = oracle.attn_prefill(q, k, v, r, w, W, R, 0.35)
    o2, _ = oracle.attn_prefill(q, k, v, r, w + 1.25, W, R, 0.35)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)


def test_window_locality(oracle):
    """Local layer: changing tokens older than the window leaves later rows bit-identical;
    changing a token inside the window changes them."""
    B, T, Hq, d, W, R = 1, 40, 2, 8, 8, 8
    q, k, v = (_rand(s, 90 + i).float() for i, s in enumerate([(B, T, Hq, d), (B, T, 1, d), (B, T, 1, d)]))
    r, w = _rand((B, T, Hq), 93).float(), _rand((Hq, R), 94).float()
    o1, l1 = oracle.attn_prefill(q, k, v, r, w, W, R, 0.3)
    k2, v2 = k.clone(), v.clone()
    k2[:, :10] += 3.0
    v2[:, :10] -= 5.0
    o2, l2 = oracle.attn_prefill(q, k2, v2, r, w, W, R, 0.3)
    first_free = 10 + W - 1  # row 17 is the first whose window starts at key 10
    assert np.array_equal(o1[:, first_free:], o2[:, first_free:])
    assert np.array_equal(l1[:, :, first_free:], l2[:, :, first_free:])
    assert not np.allclose(o1[:, first_free - 1], o2[:, first_free - 1])


def test_far_field_is_positionless(oracle):
    """Global layer: keys farther than R with equal K get exactly equal weight, so
    permuting V among them leaves the row unchanged; permuting V among near keys
    (different biases) does not."""
    T, Hq, d, R = 48, 2, 48, 8
    i = T - 1
    far = list(range(0, i - R + 1))   # distances >= R
    q = _rand((1, T, Hq, d), 100).float()
    k = _rand((1, T, 1, d), 101).float()
    k[0, far] = k[0, 0].clone()
    v = torch.eye(T).reshape(1, T, 1, d)          # read the weights out
    r, w = _rand((1, T, Hq), 102).float(), _rand((Hq, R), 103).float()
    o, _ = oracle.attn_prefill(q, k, v, r, w, 0, R, 0.2, rows=[(0, h, i) for h in range(Hq)])
    for h in range(Hq):
        pf = o[h, far]
        assert np.max(np.abs(pf - pf[0])) <= 1e-15 * max(1.0, abs(pf[0]))
        near = o[h, i - R + 1:i + 1]
        assert np.ptp(near) > 1e-6
    vv = _rand((1, T, 1, d), 104).float()
    perm = torch.arange(T)
    perm[far] = torch.tensor(far)[torch.randperm(len(far), generator=torch.Generator().manual_seed(5))]
    o1, _ = oracle.attn_prefill(q, k, vv, r, w, 0, R, 0.2, rows=[(0, 0, i)])
    o2, _ = oracle.attn_prefill(q, k, vv[:, perm], r, w, 0, R, 0.2, rows=[(0, 0, i)])
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    perm_near = torch.arange(T)
    perm_near[i - 3], perm_near[i - 1] = i - 1, i - 3
    o3, _ = oracle.attn_prefill(q, k, vv[:, perm_near], r, w, 0, R, 0.2, rows=[(0, 0, i)])
    assert not np.allclose(o1, o3)


def test_window_one_returns_own_value(oracle):
    T, Hq, d = 9, 2, 4
    v = _rand((1, T, 1, d), 110).float()
    o, lse = oracle.attn_prefill(_rand((1, T, Hq, d), 111).float(), _rand((1, T, 1, d), 112).float(), v,
                                 _rand((1, T, Hq), 113).float(), _rand((Hq, 3), 114).float(), 1, 3, 0.5)
    np.testing.assert_allclose(o[0, :, 0], v.double().numpy()[0, :, 0], rtol=0, atol=0)


def test_r_range_zero_is_nope(oracle):
    """R = 0: no distance carries a bias."""
    B, T, Hq, d = 1, 15, 2, 4
    q, k, v = (_rand(s, 120 + i).float().double() for i, s in enumerate([(B, T, Hq, d), (B, T, 1, d), (B, T, 1, d)]))
    o, _ = oracle.attn_prefill(q, k, v, _rand((B, T, Hq), 123).float(), torch.zeros(Hq, 0), 0, 0, 0.5)
    np.testing.assert_allclose(o, _sdpa(q, k, v, 0.5, 0).numpy(), rtol=0, atol=1e-12)


def test_decode_is_last_prefill_row(oracle):
    B, N, Hq, Hkv, d, R = 2, 50, 4, 2, 8, 12
    q, k, v = (_rand(s, 130 + i).float() for i, s in enumerate([(B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, d)]))
    r, w = _rand((B, N, Hq), 133).float(), _rand((Hq, R), 134).float()
    o, lse = oracle.attn_prefill(q, k, v, r, w, 0, R, 0.3)
    od, ld = oracle.attn_decode(q[:, -1], k, v, r[:, -1], w, 0, R, 0.3)
    np.testing.assert_array_equal(od, o[:, -1])
    np.testing.assert_array_equal(ld, lse[:, :, -1])


def test_rejects_bad_arguments(oracle):
    q = torch.zeros(1, 4, 3, 2)
    k = torch.zeros(1, 4, 2, 2)
    with pytest.raises(ValueError):   # 3 query heads on 2 key/value heads
        oracle.attn_prefill(q, k, k, torch.zeros(1, 4, 3), torch.zeros(3, 2), 0, 2, 1.0)
    with pytest.raises(ValueError):   # row index past the end
        oracle.attn_prefill(torch.zeros(1, 4, 2, 2), k, k, torch.zeros(1, 4, 2), torch.zeros(2, 2), 0, 2, 1.0,
                            rows=[(0, 0, 4)])


# --- context-length temperature (the essay's "The temperature scale is dependent on
# context length" section; reading: tau(n) = max(1, ln n / ln n0), n = keys the query sees)


def test_temperature_off_is_identity(oracle):
    """No break point, or a break point no row's key count exceeds, changes nothing."""
    B, T, Hq, Hkv, d, R = 1, 70, 4, 2, 8, 16
    q, k, v = (_rand(s, 150 + i).float() for i, s in enumerate([(B, T, Hq, d), (B, T, Hkv, d), (B, T, Hkv, d)]))
    r, w = _rand((B, T, Hq), 153).float(), _rand((Hq, R), 154).float()
    for window in (0, 32):
        o0, l0 = oracle.attn_prefill(q, k, v, r, w, window, R, 0.3)
        for n0 in (1, T, T + 5):
            o1, l1 = oracle.attn_prefill(q, k, v, r, w, window, R, 0.3, temp_n0=n0)
            np.testing.assert_array_equal(o1, o0)
            np.testing.assert_array_equal(l1, l0)


def test_temperature_at_square_of_break_point_doubles_logits(oracle):
    """A row that sees n0^2 keys has tau = 2: the same as doubling both the scale and
    the bias table without a temperature (the page scales the queries and the bias)."""
    B, T, Hq, Hkv, d, R, n0 = 1, 90, 4, 2, 8, 24, 8
    q, k, v = (_rand(s, 160 + i).float() for i, s in enumerate([(B, T, Hq, d), (B, T, Hkv, d), (B, T, Hkv, d)]))
    r, w = _rand((B, T, Hq), 163).float(), _rand((Hq, R), 164).float()
    # causal: row 63 sees exactly 64 keys; window 64: every row from 63 on does
    for window, rows_i in ((0, [63]), (64, list(range(63, T)))):
        rows = [(0, h, i) for h in range(Hq) for i in rows_i]
        o_t, l_t = oracle.attn_prefill(q, k, v, r, w, window, R, 0.3, rows=rows, temp_n0=n0)
        o_2, l_2 = oracle.attn_prefill(q, k, v, r, 2 * w, window, R, 0.6, rows=rows)
        np.testing.assert_allclose(o_t, o_2, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(l_t, l_2, rtol=1e-12, atol=1e-12)


def test_temperature_without_bias_is_sdpa_with_scaled_queries(oracle):
    """With r = 0 the temperature multiplies each query row: torch SDPA on q * tau_i."""
    B, T, Hq, Hkv, d, R, n0 = 2, 100, 4, 2, 16, 8, 16
    q, k, v = _rand((B, T, Hq, d), 170), _rand((B, T, Hkv, d), 171), _rand((B, T, Hkv, d), 172)
    r = torch.zeros(B, T, Hq, dtype=torch.float64)
    w = _rand((Hq, R), 173)
    for window in (0, 40):
        n = torch.tensor([len(_attended(i, window)) for i in range(T)], dtype=torch.float64)
        tau = torch.clamp(torch.log(n) / math.log(n0), min=1.0)
        # the oracle reads float32 inputs: give SDPA the same values
        qf, kf, vf = (x.float().double() for x in (q, k, v))
        ref = _sdpa(qf * tau[None, :, None, None], kf, vf, 0.25, window)
        o, _ = oracle.attn_prefill(qf, kf, vf, r, w, window, R, 0.25, temp_n0=n0)
        np.testing.assert_allclose(o, ref.numpy(), rtol=1e-10, atol=1e-10)


def test_temperature_decode_matches_prefill_row(oracle):
    B, N, Hq, Hkv, d, R, n0 = 2, 60, 4, 2, 8, 12, 10
    q, k, v = (_rand(s, 180 + i).float() for i, s in enumerate([(B, N, Hq, d), (B, N, Hkv, d), (B, N, Hkv, d)]))
    r, w = _rand((B, N, Hq), 183).float(), _rand((Hq, R), 184).float()
    o, lse = oracle.attn_prefill(q, k, v, r, w, 0, R, 0.3, temp_n0=n0)
    od, ld = oracle.attn_decode(q[:, -1], k, v, r[:, -1], w, 0, R, 0.3, temp_n0=n0)
    np.testing.assert_array_equal(od, o[:, -1])
    np.testing.assert_array_equal(ld, lse[:, :, -1])
