"""The Python binding checks tensor shapes and dtypes before anything reaches the
library (no GPU needed: these calls fail on the host with ValueError)."""
import pytest
import torch

from attention_learned_relative_b200 import ops


def _t(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype)


def test_bank_prefill_rejects_a_table_of_the_wrong_shape():
    q = _t(1, 8, 4, 64)
    kv = _t(1, 8, 2, 64)
    rs = _t(1, 8, 4, 16)
    with pytest.raises(ValueError):
        ops.attn_fwd_bank(q, kv, kv, rs, _t(1, 8, 32), 0, 32)      # C of proj != C of rs
    with pytest.raises(ValueError):
        ops.attn_fwd_bank(q, kv, kv, rs, _t(3, 16, 32), 0, 32)     # proj_heads neither 1 nor Hq
    with pytest.raises(ValueError):
        ops.attn_fwd_bank(q, kv, kv, _t(1, 8, 4), _t(1, 16, 32), 0, 32)   # rs without a C axis


def test_bank_decode_rejects_coefficients_of_the_wrong_shape():
    q = _t(2, 8, 128, dtype=torch.bfloat16)
    cache = _t(2, 100, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.attn_decode_bank(q, cache, cache, _t(2, 4, 16), _t(1, 16, 64), 0, 64)   # rs heads != Hq


def test_backward_rejects_mismatched_shapes():
    q = _t(1, 8, 4, 64)
    kv = _t(1, 8, 2, 64)
    r = _t(1, 8, 4)
    w = _t(4, 16)
    lse = _t(1, 4, 8)
    with pytest.raises(ValueError):
        ops.attn_bwd(q, kv, kv, r, w, _t(1, 8, 4, 32), lse, q, 0, 16)       # o not shaped like q
    with pytest.raises(ValueError):
        ops.attn_bwd(q, kv, kv, r, w, q, _t(1, 8, 4), q, 0, 16)             # lse transposed
    with pytest.raises(ValueError):
        ops.attn_bwd(q, kv, kv, r, w, q.bfloat16(), lse, q, 0, 16)          # mixed dtypes
