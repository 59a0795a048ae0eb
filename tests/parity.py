"""Shared helpers of the GPU parity tests: tolerances and comparisons against the
fp64 oracle.

Tolerances (stated for the method's two storage types):
* bf16 inputs, fp32 accumulation: max |O - O_ref| <= 2e-2 and mean |O - O_ref| <= 2e-3
  over every compared element, plus |LSE - LSE_ref| <= 2e-2 per row.  Also the largest
  per-row relative error, max_c |O - O_ref| / max_c |O_ref| over each row, which stays
  meaningful where long-context outputs shrink toward the mean of V and absolute bounds
  say little: <= 2e-2 (bf16 output rounding is 2^-9 relative; P in bf16 adds less).
* fp32: max |O - O_ref| <= 1e-5 * max(1e-3, max |O_ref|), LSE within 1e-5 relative.
"""
import numpy as np
import torch

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
BF16_LSE_ABS = 2e-2
BF16_ROW_REL = 2e-2
FP32_REL = 1e-5


def assert_bf16_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    o = o_gpu.detach().float().cpu().double().numpy() if hasattr(o_gpu, "detach") else np.asarray(o_gpu)
    ref = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(o - ref)
    assert np.isfinite(o).all(), what + ": non-finite output"
    assert err.max() <= BF16_MAX_ABS, "%s: max abs err %.3e" % (what, err.max())
    assert err.mean() <= BF16_MEAN_ABS, "%s: mean abs err %.3e" % (what, err.mean())
    rows_err = err.reshape(-1, err.shape[-1]).max(axis=1)
    rows_ref = np.abs(ref).reshape(-1, ref.shape[-1]).max(axis=1)
    row_rel = float((rows_err / np.maximum(rows_ref, 1e-30)).max())
    print("%s: max abs %.3e, mean abs %.3e, max row-relative %.3e" % (what, err.max(), err.mean(), row_rel))
    assert row_rel <= BF16_ROW_REL, "%s: max row-relative err %.3e" % (what, row_rel)
    if lse_gpu is not None:
        lg = lse_gpu.detach().cpu().double().numpy() if hasattr(lse_gpu, "detach") else np.asarray(lse_gpu)
        le = np.abs(lg - np.asarray(lse_ref, dtype=np.float64))
        assert le.max() <= BF16_LSE_ABS, "%s: lse max abs err %.3e" % (what, le.max())
    return float(err.max()), float(err.mean())


def assert_fp32_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    o = o_gpu.detach().cpu().double().numpy()
    ref = np.asarray(o_ref, dtype=np.float64)
    tol = FP32_REL * max(1e-3, float(np.abs(ref).max()))
    err = float(np.abs(o - ref).max())
    assert err <= tol, "%s: max abs err %.3e > %.3e" % (what, err, tol)
    if lse_gpu is not None:
        lg = lse_gpu.detach().cpu().double().numpy()
        lr = np.asarray(lse_ref, dtype=np.float64)
        assert np.abs(lg - lr).max() <= FP32_REL * max(1.0, float(np.abs(lr).max())), what + ": lse"
    return err


def sample_rows(B, T, Hq, per_head, seed, extra=()):
    """(b, h, i) rows: tile edges and bias / window boundaries plus seeded random rows."""
    g = torch.Generator().manual_seed(seed)
    fixed = {0, 1, 63, 64, 127, 128, 129, 255, 256, 511, 512, 513, 1023, 1024, 1025, T - 2, T - 1}
    fixed |= set(extra)
    fixed = sorted(i for i in fixed if 0 <= i < T)
    rows = []
    for b in range(B):
        for h in range(Hq):
            rnd = torch.randint(0, T, (per_head,), generator=g).tolist()
            for i in sorted(set(fixed) | set(rnd)):
                rows.append((b, h, i))
    return np.array(rows, dtype=np.int64)
