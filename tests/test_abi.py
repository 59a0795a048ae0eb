"""The C ABI without a GPU: the library loads, exports every function that
include/relbias_attn.h declares, and rejects bad arguments on the host (no CUDA
call is made before the checks pass)."""
import ctypes
import os
import re

import pytest

from attention_learned_relative_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "relbias_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^RELBIAS_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for want in ["relbias_attn_fwd", "relbias_attn_decode", "relbias_attn_decode_workspace_size",
                 "relbias_last_error", "relbias_device_status", "relbias_version"]:
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(ops.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), name
        assert name in ops.SIGNATURES, "binding lacks " + name


def test_binding_argument_counts_match_header():
    """Every declaration's parameter count equals the binding's argtypes (catches ABI drift)."""
    text = open(HEADER).read()
    for m in re.finditer(r"^RELBIAS_API\s+[\w\s\*]*?\b(\w+)\s*\(([^)]*)\)", text, flags=re.M):
        name, params = m.group(1), m.group(2).strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(ops.SIGNATURES[name][1]) == n, (name, n, len(ops.SIGNATURES[name][1]))


def test_version(lib):
    assert ops.version() >= 600


def test_fwd_bank_workspace_size(lib):
    # bf16: [B, T, Hq] rows of R + 14 floats rounded up to 8, rounded up to 256 bytes; fp32: none.
    stride = (16 + 14 + 7) // 8 * 8
    want = (2 * 10 * 4 * stride * 4 + 255) // 256 * 256
    assert ops.fwd_bank_workspace_size(2, 10, 4, 16, ops.RELBIAS_BF16) == want
    assert ops.fwd_bank_workspace_size(2, 10, 4, 16, ops.RELBIAS_FP32) == 0
    assert ops.fwd_bank_workspace_size(2, 10, 4, 0, ops.RELBIAS_BF16) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails its checks first


def _fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=None, B=1, T=8, Hq=4, Hkv=2, d=128,
             window=0, R=16, scale=0.125, temp_n0=0, dtype=ops.RELBIAS_BF16)
    a.update(kw)
    return lib.relbias_attn_fwd(a["q"], a["k"], a["v"], a["r"], a["w"], a["o"], a["lse"], a["B"], a["T"],
                                a["Hq"], a["Hkv"], a["d"], a["window"], a["R"], a["scale"], a["temp_n0"],
                                a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), ops.RELBIAS_ERR_ARG),
    (dict(Hkv=0), ops.RELBIAS_ERR_ARG),
    (dict(B=-1), ops.RELBIAS_ERR_ARG),
    (dict(R=-1), ops.RELBIAS_ERR_ARG),
    (dict(scale=0.0), ops.RELBIAS_ERR_ARG),
    (dict(scale=float("inf")), ops.RELBIAS_ERR_ARG),
    (dict(scale=float("nan")), ops.RELBIAS_ERR_ARG),
    (dict(q=None), ops.RELBIAS_ERR_ARG),
    (dict(w=None), ops.RELBIAS_ERR_ARG),
    (dict(o=FAKE + 8), ops.RELBIAS_ERR_ARG),
    (dict(k=FAKE + 2), ops.RELBIAS_ERR_ARG),
    (dict(r=FAKE + 1), ops.RELBIAS_ERR_ARG),
    (dict(dtype=7), ops.RELBIAS_ERR_ARG),
    (dict(d=96), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(R=4096), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(d=48, dtype=ops.RELBIAS_FP32), ops.RELBIAS_ERR_UNSUPPORTED),
])
def test_fwd_rejects_on_host(lib, kw, code):
    assert _fwd(lib, **kw) == code
    assert ops.last_error() != ""


def test_empty_inputs_are_a_no_op(lib):
    assert _fwd(lib, B=0) == ops.RELBIAS_OK
    assert _fwd(lib, T=0) == ops.RELBIAS_OK
    assert _fwd(lib, B=0, q=None, k=None, v=None, o=None, r=None) == ops.RELBIAS_OK
    assert ops.last_error() == ""


def test_r0_needs_no_table(lib):
    # R == 0 with w == NULL passes the argument checks (it then fails only for the
    # missing device on a CPU-only host, or runs on a GPU host).
    rc = _fwd(lib, R=0, w=None, d=96)
    assert rc == ops.RELBIAS_ERR_UNSUPPORTED


def _dec(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=None, B=2, N=100, Hq=8, Hkv=1, d=128,
             window=0, R=16, scale=0.1, temp_n0=0, dtype=ops.RELBIAS_BF16, ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    return lib.relbias_attn_decode(a["q"], a["k"], a["v"], a["r"], a["w"], a["o"], a["lse"], a["B"], a["N"],
                                   a["Hq"], a["Hkv"], a["d"], a["window"], a["R"], a["scale"], a["temp_n0"],
                                   a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), ops.RELBIAS_ERR_ARG),
    (dict(ws=None), ops.RELBIAS_ERR_ARG),
    (dict(ws=FAKE + 4), ops.RELBIAS_ERR_ARG),
    (dict(Hq=12, Hkv=8), ops.RELBIAS_ERR_ARG),
    (dict(scale=-1.0), ops.RELBIAS_ERR_ARG),
    (dict(dtype=ops.RELBIAS_FP32), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(d=64), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(Hq=16, Hkv=1), ops.RELBIAS_ERR_UNSUPPORTED),
])
def test_decode_rejects_on_host(lib, kw, code):
    assert _dec(lib, **kw) == code
    assert ops.last_error() != ""


def test_decode_empty_batch(lib):
    assert _dec(lib, B=0) == ops.RELBIAS_OK


def test_workspace_size_rejects_bad_shapes(lib):
    assert ops.decode_workspace_size(0, 8, 1, 100, 128, 0) == 0
    assert ops.decode_workspace_size(1, 8, 3, 100, 128, 0) == 0


def _paged(lib, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=None, B=2, num_pages=10,
             page_size=64, max_pages=5, max_seq_len=300, Hq=8, Hkv=2, d=128, window=0, R=16, scale=0.1, temp_n0=0,
             dtype=ops.RELBIAS_BF16, ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    return lib.relbias_attn_decode_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["r"], a["w"], a["o"],
                                         a["lse"], a["B"], a["num_pages"], a["page_size"], a["max_pages"],
                                         a["max_seq_len"], a["Hq"], a["Hkv"], a["d"], a["window"], a["R"],
                                         a["scale"], a["temp_n0"], a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(page_size=48), ops.RELBIAS_ERR_ARG),          # not a multiple of 32
    (dict(page_size=0), ops.RELBIAS_ERR_ARG),
    (dict(max_pages=4), ops.RELBIAS_ERR_ARG),           # 4 * 64 < max_seq_len 300
    (dict(num_pages=0), ops.RELBIAS_ERR_ARG),
    (dict(max_seq_len=0), ops.RELBIAS_ERR_ARG),
    (dict(bt=None), ops.RELBIAS_ERR_ARG),
    (dict(sl=None), ops.RELBIAS_ERR_ARG),
    (dict(sl=FAKE + 2), ops.RELBIAS_ERR_ARG),           # misaligned
    (dict(Hq=9), ops.RELBIAS_ERR_ARG),
])
def test_paged_decode_rejects_bad_arguments(lib, kw, code):
    assert _paged(lib, **kw) == code
    assert ops.last_error() != ""


def test_paged_decode_batch_zero_is_a_no_op(lib):
    assert _paged(lib, B=0) == ops.RELBIAS_OK


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=None, B=1, T=8, q_off=16, kv_T=24, Hq=4, Hkv=2,
             d=128, window=0, R=16, scale=0.125, temp_n0=0, dtype=ops.RELBIAS_BF16)
    a.update(kw)
    return lib.relbias_attn_fwd_chunk(a["q"], a["k"], a["v"], a["r"], a["w"], a["o"], a["lse"], a["B"], a["T"],
                                      a["q_off"], a["kv_T"], a["Hq"], a["Hkv"], a["d"], a["window"], a["R"],
                                      a["scale"], a["temp_n0"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q_off=-1), ops.RELBIAS_ERR_ARG),
    (dict(q_off=17), ops.RELBIAS_ERR_ARG),          # q_off + T > kv_T
    (dict(kv_T=0), ops.RELBIAS_ERR_ARG),
    (dict(Hq=3), ops.RELBIAS_ERR_ARG),
    (dict(k=FAKE + 2), ops.RELBIAS_ERR_ARG),
    (dict(d=96), ops.RELBIAS_ERR_UNSUPPORTED),
])
def test_chunk_rejects_on_host(lib, kw, code):
    assert _chunk(lib, **kw) == code
    assert ops.last_error() != ""


def test_chunk_empty_is_a_no_op(lib):
    assert _chunk(lib, T=0) == ops.RELBIAS_OK
    assert _chunk(lib, B=0) == ops.RELBIAS_OK


def _fwd_bank(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, rs=FAKE, proj=FAKE, o=FAKE, lse=None, B=1, T=8, Hq=4, Hkv=2, d=64, C=16,
             proj_heads=1, window=0, R=16, scale=0.125, temp_n0=0, dtype=ops.RELBIAS_FP32, ws=None, ws_bytes=0)
    a.update(kw)
    return lib.relbias_attn_fwd_bank(a["q"], a["k"], a["v"], a["rs"], a["proj"], a["o"], a["lse"], a["B"], a["T"],
                                     a["Hq"], a["Hkv"], a["d"], a["C"], a["proj_heads"], a["window"], a["R"],
                                     a["scale"], a["temp_n0"], a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(C=0), ops.RELBIAS_ERR_ARG),
    (dict(C=17), ops.RELBIAS_ERR_ARG),
    (dict(proj_heads=2), ops.RELBIAS_ERR_ARG),       # neither 1 nor Hq
    (dict(rs=None), ops.RELBIAS_ERR_ARG),
    (dict(proj=None), ops.RELBIAS_ERR_ARG),
    (dict(dtype=ops.RELBIAS_BF16, d=128), ops.RELBIAS_ERR_ARG),           # bf16 bank needs its workspace
    (dict(dtype=ops.RELBIAS_BF16, d=128, ws=FAKE + 16, ws_bytes=1 << 20), ops.RELBIAS_ERR_ARG),   # misaligned
    (dict(dtype=ops.RELBIAS_BF16, d=128, ws=FAKE, ws_bytes=64), ops.RELBIAS_ERR_ARG),             # too small
    (dict(dtype=ops.RELBIAS_BF16, d=96, ws=FAKE, ws_bytes=1 << 20), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(d=48), ops.RELBIAS_ERR_UNSUPPORTED),
])
def test_fwd_bank_rejects_on_host(lib, kw, code):
    assert _fwd_bank(lib, **kw) == code
    assert ops.last_error() != ""


def _dec_bank(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, rs=FAKE, proj=FAKE, o=FAKE, lse=None, B=2, N=100, Hq=8, Hkv=1, d=128, C=16,
             proj_heads=1, window=0, R=16, scale=0.1, temp_n0=0, dtype=ops.RELBIAS_BF16, ws=FAKE, ws_bytes=64)
    a.update(kw)
    return lib.relbias_attn_decode_bank(a["q"], a["k"], a["v"], a["rs"], a["proj"], a["o"], a["lse"], a["B"],
                                        a["N"], a["Hq"], a["Hkv"], a["d"], a["C"], a["proj_heads"], a["window"],
                                        a["R"], a["scale"], a["temp_n0"], a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(C=0), ops.RELBIAS_ERR_ARG),
    (dict(proj_heads=3), ops.RELBIAS_ERR_ARG),
    (dict(rs=None), ops.RELBIAS_ERR_ARG),
    (dict(ws=None), ops.RELBIAS_ERR_ARG),
    (dict(ws_bytes=64), ops.RELBIAS_ERR_ARG),          # 2*8*16 floats of curves do not fit 64 bytes
    (dict(dtype=ops.RELBIAS_FP32), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(d=64), ops.RELBIAS_ERR_UNSUPPORTED),
])
def test_decode_bank_rejects_on_host(lib, kw, code):
    assert _dec_bank(lib, **kw) == code
    assert ops.last_error() != ""


def test_decode_bank_empty_batch(lib):
    assert _dec_bank(lib, B=0) == ops.RELBIAS_OK


def _bwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, dr=FAKE,
             dw=FAKE, B=1, T=8, Hq=4, Hkv=2, d=64, window=0, R=16, scale=0.125, temp_n0=0, dtype=ops.RELBIAS_BF16,
             ws=FAKE, ws_bytes=16)
    a.update(kw)
    return lib.relbias_attn_bwd(a["q"], a["k"], a["v"], a["r"], a["w"], a["o"], a["lse"], a["dout"], a["dq"], a["dk"],
                                a["dv"], a["dr"], a["dw"], a["B"], a["T"], a["Hq"], a["Hkv"], a["d"], a["window"],
                                a["R"], a["scale"], a["temp_n0"], a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(lse=None), ops.RELBIAS_ERR_ARG),
    (dict(dw=None), ops.RELBIAS_ERR_ARG),             # R > 0 needs dw
    (dict(dout=FAKE + 4), ops.RELBIAS_ERR_ARG),
    (dict(Hq=3), ops.RELBIAS_ERR_ARG),
    (dict(dtype=5), ops.RELBIAS_ERR_ARG),
    (dict(d=96), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(R=40000), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(ws_bytes=16), ops.RELBIAS_ERR_ARG),          # B*Hq*T floats = 128 bytes needed
])
def test_bwd_rejects_on_host(lib, kw, code):
    assert _bwd(lib, **kw) == code
    assert ops.last_error() != ""


def test_bwd_empty_and_workspace_size(lib):
    assert _bwd(lib, T=0) == ops.RELBIAS_OK
    assert ops.lib().relbias_attn_bwd_workspace_size(2, 100, 8) == 2 * 100 * 8 * 4
    assert ops.lib().relbias_attn_bwd_workspace_size(0, 100, 8) == 16


def _dec_noalloc(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=None, B=2, N=100, Hq=8, Hkv=1, d=128,
             window=0, R=16, scale=0.1, temp_n0=0, dtype=ops.RELBIAS_BF16)
    a.update(kw)
    return lib.relbias_attn_decode_noalloc(a["q"], a["k"], a["v"], a["r"], a["w"], a["o"], a["lse"], a["B"],
                                           a["N"], a["Hq"], a["Hkv"], a["d"], a["window"], a["R"], a["scale"],
                                           a["temp_n0"], a["dtype"], None)


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(r=None), dict(o=FAKE + 8), dict(k=FAKE + 2), dict(lse=FAKE + 1), dict(N=0),
    dict(Hq=12, Hkv=8), dict(scale=0.0), dict(R=-1), dict(w=None), dict(dtype=9),
    dict(dtype=ops.RELBIAS_FP32), dict(d=64), dict(Hq=16, Hkv=1),
    dict(),   # valid arguments: both then fail alike at the device query on a host without a GPU
])
def test_noalloc_reports_argument_errors_like_the_regular_decode(lib, kw):
    """The allocation-free decode checks its arguments before it looks up its static
    scratch, and reports them with the regular entry point's code and message."""
    rc_ref = _dec(lib, **kw)
    msg_ref = ops.last_error()
    rc = _dec_noalloc(lib, **kw)
    assert rc == rc_ref
    assert ops.last_error() == msg_ref
    if kw:
        assert rc in (ops.RELBIAS_ERR_ARG, ops.RELBIAS_ERR_UNSUPPORTED)


def test_noalloc_empty_batch(lib):
    assert _dec_noalloc(lib, B=0) == ops.RELBIAS_OK
    assert _dec_noalloc(lib, B=0, q=None, o=None) == ops.RELBIAS_OK


def _chunk_paged(lib, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, qo=FAKE, ql=FAKE, r=FAKE, w=FAKE, o=FAKE, lse=None, B=2, T=100,
             num_pages=8, page_size=128, max_pages=4, Hq=8, Hkv=2, d=128, window=0, R=64, scale=0.1, temp_n0=0,
             dtype=ops.RELBIAS_BF16)
    a.update(kw)
    return lib.relbias_attn_fwd_chunk_paged(a["q"], a["kp"], a["vp"], a["bt"], a["qo"], a["ql"], a["r"], a["w"],
                                            a["o"], a["lse"], a["B"], a["T"], a["num_pages"], a["page_size"],
                                            a["max_pages"], a["Hq"], a["Hkv"], a["d"], a["window"], a["R"],
                                            a["scale"], a["temp_n0"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(page_size=96), ops.RELBIAS_ERR_ARG),           # not a multiple of 64
    (dict(page_size=0), ops.RELBIAS_ERR_ARG),
    (dict(num_pages=0), ops.RELBIAS_ERR_ARG),
    (dict(max_pages=0), ops.RELBIAS_ERR_ARG),
    (dict(bt=None), ops.RELBIAS_ERR_ARG),
    (dict(qo=None), ops.RELBIAS_ERR_ARG),
    (dict(ql=FAKE + 2), ops.RELBIAS_ERR_ARG),            # misaligned
    (dict(kp=FAKE + 8), ops.RELBIAS_ERR_ARG),
    (dict(Hq=9), ops.RELBIAS_ERR_ARG),
    (dict(dtype=ops.RELBIAS_FP32), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(d=96), ops.RELBIAS_ERR_UNSUPPORTED),
    (dict(R=4096), ops.RELBIAS_ERR_UNSUPPORTED),
])
def test_chunk_paged_rejects_on_host(lib, kw, code):
    assert _chunk_paged(lib, **kw) == code
    assert ops.last_error() != ""


def test_chunk_paged_empty_is_a_no_op(lib):
    assert _chunk_paged(lib, B=0) == ops.RELBIAS_OK
    assert _chunk_paged(lib, T=0) == ops.RELBIAS_OK
