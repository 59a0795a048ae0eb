"""Python binding of librelbias_attn.so (ctypes).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and their device pointers passed to the C entry points declared in
include/relbias_attn.h.  Every step of the computation runs in the library's CUDA
kernels; there is no fallback path.  If the shared library is missing the calls
raise, they never compute anything on the CPU.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librelbias_attn.so")

RELBIAS_OK = 0
RELBIAS_ERR_ARG = -1
RELBIAS_ERR_UNSUPPORTED = -2
RELBIAS_ERR_CUDA = -3
RELBIAS_STATUS_TIMEOUT = 1
RELBIAS_STATUS_BAD_LENGTH = 2
RELBIAS_BF16 = 0
RELBIAS_FP32 = 1

# Every symbol include/relbias_attn.h declares: (name, restype, argtypes).
_VP = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "relbias_attn_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "relbias_attn_fwd_chunk": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                    _I, _VP]),
    "relbias_attn_fwd_chunk_paged": (_I, [_VP] * 10 + [_I] * 10 + [_F, _I, _I, _VP]),
    "relbias_attn_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "relbias_attn_decode": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP,
                                 _SZ, _VP]),
    "relbias_attn_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                         _I, _VP]),
    "relbias_attn_decode_paged_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "relbias_attn_decode_paged": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I,
                                       _I, _I, _F, _I, _I, _VP, _SZ, _VP]),
    "relbias_attn_fwd_bank_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "relbias_attn_fwd_bank": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                   _I, _VP, _SZ, _VP]),
    "relbias_attn_decode_bank_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "relbias_attn_decode_bank": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                      _I, _VP, _SZ, _VP]),
    "relbias_attn_bwd_workspace_size": (_SZ, [_I, _I, _I]),
    "relbias_attn_bwd": (_I, [_VP] * 13 + [_I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP, _SZ, _VP]),
    "relbias_attn_bwd_bank_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "relbias_attn_bwd_bank": (_I, [_VP] * 13 + [_I] * 9 + [_F, _I, _I, _VP, _SZ, _VP]),
    "relbias_last_error": (ctypes.c_char_p, []),
    "relbias_device_status": (_I, [_I]),
    "relbias_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "relbias_version": (_I, []),
}

_lib = None


class RelbiasError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("relbias error %d: %s" % (code, msg))
        self.code = code


def lib():
    """The loaded shared library (built in-tree by attention_learned_relative_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("%s is missing: build it with `python -m attention_learned_relative_b200.build`"
                               % LIB_PATH)
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _check(rc: int):
    if rc != RELBIAS_OK:
        raise RelbiasError(rc, lib().relbias_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return RELBIAS_BF16
    if t.dtype == torch.float32:
        return RELBIAS_FP32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def attn_fwd(q, k, v, r, w, window: int, R: int, scale: float | None = None, out=None, lse=None,
             stream=None, temp_n0: int = 0):
    """Prefill.  q [B,T,Hq,d], k/v [B,T,Hkv,d] (bf16 or fp32, CUDA, contiguous),
    r [B,T,Hq] fp32, w [Hq,R] fp32.  Returns o [B,T,Hq,d] (and fills `lse`
    [B,Hq,T] fp32 when given).  scale defaults to 1/sqrt(d).  temp_n0 > 1 applies
    the context-length temperature max(1, ln n / ln temp_n0) to the logits of a row
    that sees n keys (see include/relbias_attn.h)."""
    _need(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,T,Hq,d], k/v [B,T,Hkv,d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(k.shape[:2] == (B, T) and k.shape[3] == d, "k/v shape %s does not match q %s" % (k.shape, q.shape))
    _need(q.dtype == k.dtype == v.dtype, "q, k, v must share a dtype")
    _need(r.shape == (B, T, Hq) and r.dtype == torch.float32, "r must be fp32 [B,T,Hq]")
    _need(w is None or (w.shape == (Hq, R) and w.dtype == torch.float32), "w must be fp32 [Hq,R]")
    for t in (q, k, v, r, w, out, lse):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(out.shape == q.shape and out.dtype == q.dtype, "out must match q")
    _need(lse is None or (lse.shape == (B, Hq, T) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq,T]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(w), _ptr(out), _ptr(lse),
                                B, T, Hq, Hkv, d, int(window), int(R), float(scale), int(temp_n0),
                                _dtype_code(q), _stream_handle(stream, q.device))
    _check(rc)
    return out


def attn_fwd_chunk(q, k, v, r, w, q_off: int, window: int, R: int, scale: float | None = None, out=None,
                   lse=None, stream=None, temp_n0: int = 0):
    """Chunked prefill: the T rows of q [B,T,Hq,d] sit at positions q_off ... q_off+T-1
    and attend to the cache k/v [B,kv_T,Hkv,d] (kv_T >= q_off+T; rows q_off ... q_off+T-1
    are the chunk's own keys and values).  r [B,T,Hq] fp32, w [Hq,R] fp32.  Returns
    o [B,T,Hq,d] (fills `lse` [B,Hq,T] when given)."""
    _need(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,T,Hq,d], k/v [B,kv_T,Hkv,d]")
    B, T, Hq, d = q.shape
    kv_T, Hkv = k.shape[1], k.shape[2]
    _need(k.shape[0] == B and k.shape[3] == d, "k/v shape %s does not match q %s" % (k.shape, q.shape))
    _need(q.dtype == k.dtype == v.dtype, "q, k, v must share a dtype")
    _need(r.shape == (B, T, Hq) and r.dtype == torch.float32, "r must be fp32 [B,T,Hq]")
    _need(w is None or (w.shape == (Hq, R) and w.dtype == torch.float32), "w must be fp32 [Hq,R]")
    for t in (q, k, v, r, w, out, lse):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(out.shape == q.shape and out.dtype == q.dtype, "out must match q")
    _need(lse is None or (lse.shape == (B, Hq, T) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq,T]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_fwd_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(w), _ptr(out), _ptr(lse),
                                      B, T, int(q_off), kv_T, Hq, Hkv, d, int(window), int(R), float(scale),
                                      int(temp_n0), _dtype_code(q), _stream_handle(stream, q.device))
    _check(rc)
    return out


def attn_fwd_chunk_paged(q, k_pages, v_pages, block_table, q_offs, q_lens, r, w, window: int, R: int,
                         scale: float | None = None, out=None, lse=None, stream=None, temp_n0: int = 0):
    """Chunked prefill against a paged cache.  q [B,T,Hq,d] bf16 (sequence b's chunk is
    its first q_lens[b] rows, at positions q_offs[b] ...), k_pages/v_pages
    [num_pages,page_size,Hkv,d] bf16, block_table [B,max_pages] int32, q_offs/q_lens [B]
    int32, r [B,T,Hq] fp32, w [Hq,R] fp32.  Returns o [B,T,Hq,d]; rows at or past
    q_lens[b] are left as they were in `out` (allocated, uninitialised, if None)."""
    _need(q.dim() == 4 and k_pages.dim() == 4 and v_pages.shape == k_pages.shape,
          "q [B,T,Hq,d], pages [num_pages,page_size,Hkv,d]")
    B, T, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_pages.shape
    _need(dk == d, "page head dim %d != q head dim %d" % (dk, d))
    _need(q.dtype == k_pages.dtype == v_pages.dtype, "q and pages must share a dtype")
    _need(block_table.dim() == 2 and block_table.shape[0] == B and block_table.dtype == torch.int32,
          "block_table must be int32 [B, max_pages]")
    for name, t_ in (("q_offs", q_offs), ("q_lens", q_lens)):
        _need(t_.shape == (B,) and t_.dtype == torch.int32, "%s must be int32 [B]" % name)
    _need(r.shape == (B, T, Hq) and r.dtype == torch.float32, "r must be fp32 [B,T,Hq]")
    _need(w is None or (w.shape == (Hq, R) and w.dtype == torch.float32), "w must be fp32 [Hq,R]")
    for t_ in (q, k_pages, v_pages, block_table, q_offs, q_lens, r, w, out, lse):
        _need(t_ is None or (t_.is_cuda and t_.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(out.shape == q.shape and out.dtype == q.dtype, "out must match q")
    _need(lse is None or (lse.shape == (B, Hq, T) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq,T]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_fwd_chunk_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(q_offs),
                                            _ptr(q_lens), _ptr(r), _ptr(w), _ptr(out), _ptr(lse), B, T, num_pages,
                                            page_size, block_table.shape[1], Hq, Hkv, d, int(window), int(R),
                                            float(scale), int(temp_n0), _dtype_code(q),
                                            _stream_handle(stream, q.device))
    _check(rc)
    return out


def decode_workspace_size(B: int, Hq: int, Hkv: int, n_ctx: int, d: int, window: int) -> int:
    """Bytes of device scratch relbias_attn_decode needs for this shape (on the current device)."""
    return int(lib().relbias_attn_decode_workspace_size(B, Hq, Hkv, n_ctx, d, int(window)))


def attn_decode(q, k_cache, v_cache, r, w, window: int, R: int, scale: float | None = None, out=None,
                lse=None, workspace=None, stream=None, temp_n0: int = 0):
    """Decode one query per sequence at position n_ctx-1.  q [B,Hq,d] bf16,
    k_cache/v_cache [B,n_ctx,Hkv,d] bf16, r [B,Hq] fp32, w [Hq,R] fp32.
    Returns o [B,Hq,d] bf16 (fills `lse` [B,Hq] when given).  `workspace` is a
    byte tensor of at least decode_workspace_size(...) bytes; allocated if None.
    temp_n0: context-length temperature break point, as for attn_fwd."""
    _need(q.dim() == 3 and k_cache.dim() == 4 and v_cache.shape == k_cache.shape, "q [B,Hq,d], cache [B,N,Hkv,d]")
    B, Hq, d = q.shape
    _, N, Hkv, _ = k_cache.shape
    _need(k_cache.shape[0] == B and k_cache.shape[3] == d, "cache shape does not match q")
    _need(q.dtype == k_cache.dtype == v_cache.dtype, "q and cache must share a dtype")
    _need(r.shape == (B, Hq) and r.dtype == torch.float32, "r must be fp32 [B,Hq]")
    _need(w is None or (w.shape == (Hq, R) and w.dtype == torch.float32), "w must be fp32 [Hq,R]")
    for t in (q, k_cache, v_cache, r, w, out, lse, workspace):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(lse is None or (lse.shape == (B, Hq) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq]")
    need = decode_workspace_size(B, Hq, Hkv, N, d, window)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(r), _ptr(w), _ptr(out), _ptr(lse),
                                   B, N, Hq, Hkv, d, int(window), int(R), float(scale), int(temp_n0),
                                   _dtype_code(q), _ptr(workspace), ws_bytes, _stream_handle(stream, q.device))
    _check(rc)
    return out


def attn_decode_noalloc(q, k_cache, v_cache, r, w, window: int, R: int, scale: float | None = None, out=None,
                        lse=None, stream=None, temp_n0: int = 0):
    """attn_decode for callers that cannot allocate device memory: the split
    partials go to the library's own static scratch (see
    relbias_attn_decode_noalloc in include/relbias_attn.h for its size limit and
    the rule that calls must not overlap on the GPU).  `out` must be given by a
    caller that cannot allocate; None allocates it here for convenience."""
    _need(q.dim() == 3 and k_cache.dim() == 4 and v_cache.shape == k_cache.shape, "q [B,Hq,d], cache [B,N,Hkv,d]")
    B, Hq, d = q.shape
    _, N, Hkv, _ = k_cache.shape
    for t in (q, k_cache, v_cache, r, w, out, lse):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(r), _ptr(w), _ptr(out),
                                           _ptr(lse), B, N, Hq, Hkv, d, int(window), int(R), float(scale),
                                           int(temp_n0), _dtype_code(q), _stream_handle(stream, q.device))
    _check(rc)
    return out


def decode_paged_workspace_size(B: int, Hq: int, Hkv: int, max_seq_len: int, d: int, window: int) -> int:
    """Bytes of device scratch relbias_attn_decode_paged needs for this shape."""
    return int(lib().relbias_attn_decode_paged_workspace_size(B, Hq, Hkv, max_seq_len, d, int(window)))


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, r, w, window: int, R: int, max_seq_len: int,
                      scale: float | None = None, out=None, lse=None, workspace=None, stream=None,
                      temp_n0: int = 0):
    """Decode against a paged, variable-length cache.  q [B,Hq,d] bf16,
    k_pages/v_pages [num_pages,page_size,Hkv,d] bf16, block_table [B,max_pages] int32,
    seq_lens [B] int32 (each in [1, max_seq_len]), r [B,Hq] fp32, w [Hq,R] fp32.
    Sequence b's query sits at position seq_lens[b]-1; its cache row t is row
    t % page_size of page block_table[b, t // page_size].  Returns o [B,Hq,d]."""
    _need(q.dim() == 3 and k_pages.dim() == 4 and v_pages.shape == k_pages.shape,
          "q [B,Hq,d], pages [num_pages,page_size,Hkv,d]")
    B, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_pages.shape
    _need(dk == d, "page head dim %d != q head dim %d" % (dk, d))
    _need(q.dtype == k_pages.dtype == v_pages.dtype, "q and pages must share a dtype")
    _need(block_table.dim() == 2 and block_table.shape[0] == B and block_table.dtype == torch.int32,
          "block_table must be int32 [B, max_pages]")
    _need(seq_lens.shape == (B,) and seq_lens.dtype == torch.int32, "seq_lens must be int32 [B]")
    _need(r.shape == (B, Hq) and r.dtype == torch.float32, "r must be fp32 [B,Hq]")
    _need(w is None or (w.shape == (Hq, R) and w.dtype == torch.float32), "w must be fp32 [Hq,R]")
    for t in (q, k_pages, v_pages, block_table, seq_lens, r, w, out, lse, workspace):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(lse is None or (lse.shape == (B, Hq) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq]")
    need = decode_paged_workspace_size(B, Hq, Hkv, max_seq_len, d, window)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                                         _ptr(r), _ptr(w), _ptr(out), _ptr(lse), B, num_pages, page_size,
                                         block_table.shape[1], int(max_seq_len), Hq, Hkv, d, int(window), int(R),
                                         float(scale), int(temp_n0), _dtype_code(q), _ptr(workspace), ws_bytes,
                                         _stream_handle(stream, q.device))
    _check(rc)
    return out


def _bank_shape(proj, C_from_rs: int, Hq: int, R: int) -> int:
    """proj_heads of a bank tensor [proj_heads, C, R] (proj_heads 1 or Hq)."""
    _need(proj is not None and proj.dim() == 3 and proj.dtype == torch.float32, "proj must be fp32 [heads,C,R]")
    _need(proj.shape[1] == C_from_rs and proj.shape[2] == R and proj.shape[0] in (1, Hq),
          "proj must be [1 or Hq, C, R] = [*, %d, %d], got %s" % (C_from_rs, R, tuple(proj.shape)))
    return int(proj.shape[0])


def fwd_bank_workspace_size(B: int, T: int, Hq: int, R: int, dtype: int) -> int:
    """Bytes of scratch attn_fwd_bank needs (0: none, for the fp32 path)."""
    return int(lib().relbias_attn_fwd_bank_workspace_size(B, T, Hq, R, dtype))


def attn_fwd_bank(q, k, v, rs, proj, window: int, R: int, scale: float | None = None, out=None, lse=None,
                  stream=None, temp_n0: int = 0, workspace=None):
    """Prefill with the shared-bank bias sum_c rs[b,i,h,c] * proj[h or 0, c, i-j].
    q [B,T,Hq,d], k/v [B,T,Hkv,d] (bf16 or fp32), rs [B,T,Hq,C] fp32,
    proj [1 or Hq, C, R] fp32.  Returns o [B,T,Hq,d].  The bf16 path writes every
    row's curve into `workspace` (a byte tensor of at least fwd_bank_workspace_size
    bytes; allocated if None) before the tensor-core kernel reads it."""
    _need(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,T,Hq,d], k/v [B,T,Hkv,d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(rs.dim() == 4 and rs.shape[:3] == (B, T, Hq) and rs.dtype == torch.float32, "rs must be fp32 [B,T,Hq,C]")
    C = int(rs.shape[3])
    proj_heads = _bank_shape(proj, C, Hq, R)
    for t in (q, k, v, rs, proj, out, lse, workspace):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(lse is None or (lse.shape == (B, Hq, T) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq,T]")
    code = _dtype_code(q)
    need = fwd_bank_workspace_size(B, T, Hq, R, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_fwd_bank(_ptr(q), _ptr(k), _ptr(v), _ptr(rs), _ptr(proj), _ptr(out), _ptr(lse),
                                     B, T, Hq, Hkv, d, C, proj_heads, int(window), int(R), float(scale),
                                     int(temp_n0), code, _ptr(workspace), ws_bytes,
                                     _stream_handle(stream, q.device))
    _check(rc)
    return out


def decode_bank_workspace_size(B: int, Hq: int, Hkv: int, n_ctx: int, d: int, window: int, R: int) -> int:
    """Bytes of scratch attn_decode_bank needs (curves plus split partials)."""
    return int(lib().relbias_attn_decode_bank_workspace_size(B, Hq, Hkv, n_ctx, d, window, R))


def attn_decode_bank(q, k_cache, v_cache, rs, proj, window: int, R: int, scale: float | None = None, out=None,
                     lse=None, workspace=None, stream=None, temp_n0: int = 0):
    """Decode with the shared-bank bias.  q [B,Hq,d] bf16, caches [B,n_ctx,Hkv,d]
    bf16, rs [B,Hq,C] fp32, proj [1 or Hq, C, R] fp32.  Returns o [B,Hq,d]."""
    _need(q.dim() == 3 and k_cache.dim() == 4 and v_cache.shape == k_cache.shape, "q [B,Hq,d], cache [B,N,Hkv,d]")
    B, Hq, d = q.shape
    _, N, Hkv, _ = k_cache.shape
    _need(rs.dim() == 3 and rs.shape[:2] == (B, Hq) and rs.dtype == torch.float32, "rs must be fp32 [B,Hq,C]")
    C = int(rs.shape[2])
    proj_heads = _bank_shape(proj, C, Hq, R)
    for t in (q, k_cache, v_cache, rs, proj, out, lse, workspace):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty_like(q)
    _need(lse is None or (lse.shape == (B, Hq) and lse.dtype == torch.float32), "lse must be fp32 [B,Hq]")
    need = decode_bank_workspace_size(B, Hq, Hkv, N, d, window, R)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_decode_bank(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(rs), _ptr(proj), _ptr(out),
                                        _ptr(lse), B, N, Hq, Hkv, d, C, proj_heads, int(window), int(R),
                                        float(scale), int(temp_n0), _dtype_code(q), _ptr(workspace), ws_bytes,
                                        _stream_handle(stream, q.device))
    _check(rc)
    return out


def attn_bwd(q, k, v, r, w, o, lse, dout, window: int, R: int, scale: float | None = None, stream=None,
             temp_n0: int = 0, workspace=None, grads=None):
    """Backward pass of attn_fwd.  q/o/dout [B,T,Hq,d], k/v [B,T,Hkv,d] (bf16 or fp32),
    r [B,T,Hq] and w [Hq,R] fp32, lse [B,Hq,T] fp32 (the forward's).  Returns a dict of
    fp32 gradients dq, dk, dv (shapes of q, k, v), dr [B,T,Hq] and dw [Hq,R] (written
    into `grads` when a dict of such tensors is given)."""
    _need(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,T,Hq,d], k/v [B,T,Hkv,d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(o.shape == q.shape and dout.shape == q.shape, "o and dout must have q's shape")
    _need(q.dtype == k.dtype == v.dtype == o.dtype == dout.dtype, "q, k, v, o, dout must share a dtype")
    _need(r.shape == (B, T, Hq) and r.dtype == torch.float32, "r must be fp32 [B,T,Hq]")
    _need(w is None or (w.shape == (Hq, R) and w.dtype == torch.float32), "w must be fp32 [Hq,R]")
    _need(lse.shape == (B, Hq, T) and lse.dtype == torch.float32, "lse must be fp32 [B,Hq,T]")
    for t in (q, k, v, r, w, o, lse, dout, workspace):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    f32 = dict(dtype=torch.float32, device=q.device)
    g = grads if grads is not None else {
        "dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32), "dv": torch.empty(v.shape, **f32),
        "dr": torch.empty(r.shape, **f32), "dw": torch.empty((Hq, max(R, 0)), **f32)}
    for name, like in (("dq", q), ("dk", k), ("dv", v), ("dr", r)):
        _need(g[name].shape == like.shape and g[name].dtype == torch.float32 and g[name].is_contiguous(),
              "%s must be a contiguous fp32 tensor of shape %s" % (name, tuple(like.shape)))
    need = int(lib().relbias_attn_bwd_workspace_size(B, T, Hq))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(w), _ptr(o), _ptr(lse), _ptr(dout),
                                _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dr"]),
                                _ptr(g["dw"]) if R > 0 else None, B, T, Hq, Hkv, d, int(window), int(R),
                                float(scale), int(temp_n0), _dtype_code(q), _ptr(workspace), ws_bytes,
                                _stream_handle(stream, q.device))
    _check(rc)
    return g



def attn_bwd_bank(q, k, v, rs, proj, o, lse, dout, window: int, R: int, scale: float | None = None, stream=None,
                  temp_n0: int = 0, workspace=None, grads=None):
    """Backward pass of attn_fwd_bank (bf16, d in {64, 128}).  rs [B,T,Hq,C] and proj
    [1 or Hq, C, R] fp32, the rest as attn_bwd.  Returns a dict of fp32 gradients dq,
    dk, dv, drs (shaped like rs) and dproj (shaped like proj), written into `grads`
    when a dict of such tensors is given."""
    _need(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,T,Hq,d], k/v [B,T,Hkv,d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _need(o.shape == q.shape and dout.shape == q.shape, "o and dout must have q's shape")
    _need(q.dtype == k.dtype == v.dtype == o.dtype == dout.dtype, "q, k, v, o, dout must share a dtype")
    _need(rs.dim() == 4 and rs.shape[:3] == (B, T, Hq) and rs.dtype == torch.float32, "rs must be fp32 [B,T,Hq,C]")
    C = int(rs.shape[3])
    proj_heads = _bank_shape(proj, C, Hq, R)
    _need(lse.shape == (B, Hq, T) and lse.dtype == torch.float32, "lse must be fp32 [B,Hq,T]")
    for t in (q, k, v, rs, proj, o, lse, dout, workspace):
        _need(t is None or (t.is_cuda and t.is_contiguous()), "tensors must be contiguous CUDA tensors")
    f32 = dict(dtype=torch.float32, device=q.device)
    g = grads if grads is not None else {
        "dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32), "dv": torch.empty(v.shape, **f32),
        "drs": torch.empty(rs.shape, **f32), "dproj": torch.empty(proj.shape, **f32)}
    for name, like in (("dq", q), ("dk", k), ("dv", v), ("drs", rs), ("dproj", proj)):
        _need(g[name].shape == like.shape and g[name].dtype == torch.float32 and g[name].is_contiguous(),
              "%s must be a contiguous fp32 tensor of shape %s" % (name, tuple(like.shape)))
    need = int(lib().relbias_attn_bwd_bank_workspace_size(B, T, Hq, R))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().relbias_attn_bwd_bank(_ptr(q), _ptr(k), _ptr(v), _ptr(rs), _ptr(proj), _ptr(o), _ptr(lse), _ptr(dout),
                                     _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["drs"]), _ptr(g["dproj"]),
                                     B, T, Hq, Hkv, d, C, proj_heads, int(window), int(R), float(scale), int(temp_n0),
                                     _dtype_code(q), _ptr(workspace), ws_bytes, _stream_handle(stream, q.device))
    _check(rc)
    return g

def device_status(reset: bool = True) -> int:
    """Synchronise and return the kernels' status bits (RELBIAS_STATUS_*)."""
    rc = lib().relbias_device_status(1 if reset else 0)
    if rc < 0:
        _check(rc)
    return rc


def set_wait_limit_ns(ns: int) -> None:
    """Bound on a single wait inside the library's kernels, in nanoseconds (0: the
    default of 2 s).  A short bound makes waits run out on purpose (failure-path tests)."""
    _check(lib().relbias_set_wait_limit_ns(int(ns)))


def last_error() -> str:
    return lib().relbias_last_error().decode()


def version() -> int:
    return int(lib().relbias_version())
