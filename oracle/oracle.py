"""fp64 CPU oracle for learned relative-position-bias attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference legs may import this module.  The product path never does: the
CUDA library and this oracle share no code.

The arithmetic lives in ``relbias_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only marshals arrays and builds that file with gcc.  The one piece
of arithmetic kept here, :func:`bias_matrix`, restates the pages' NumPy listing
for tiny inputs (the essay "Thinking Machines dropped RoPE", function
``relative_position_bias``), so a test can look at the whole (H, T, T) bias.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "relbias_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile relbias_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP).

    FMA contraction is switched off so that every product and sum is rounded
    exactly as written in the C source.
    """
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        f = lib.oracle_attn_rows
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                      ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                      ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int64,
                      ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_num_threads.restype = ctypes.c_int
        fb = lib.oracle_attn_bwd
        fb.restype = ctypes.c_int
        fb.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                       ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                       ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int64,
                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


def num_threads() -> int:
    """Number of OpenMP threads the oracle runs on."""
    return int(_load().oracle_num_threads())


def _f32(x) -> np.ndarray:
    """Any tensor or array as a C-contiguous float32 numpy array (bf16 widens exactly)."""
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def attn_rows(q_rows, rs_rows, proj, k, v, req, Hq: int, window: int, R: int, scale: float, temp_n0: int = 0):
    """Rows of biased attention.

    q_rows [n, d], rs_rows [n, C], proj [Hp, C, R] with Hp in {1, Hq},
    k, v [B, T, Hkv, d], req [n, 3] int64 of (b, h, i), Hq query heads.
    temp_n0 > 1 applies the context-length temperature tau(n) = max(1, ln n / ln temp_n0)
    to the logits of a row that sees n keys (relbias_oracle.c states the reading).
    Returns (o [n, d] float64, lse [n] float64).
    """
    lib = _load()
    q_rows = _f32(q_rows)
    rs_rows = _f32(rs_rows)
    proj = _f32(proj)
    k = _f32(k)
    v = _f32(v)
    req = np.ascontiguousarray(np.asarray(req, dtype=np.int64).reshape(-1, 3))
    n = req.shape[0]
    B, T, Hkv, d = k.shape
    if v.shape != k.shape:
        raise ValueError("k and v shapes differ")
    _, C, Rt = proj.shape
    if Rt != R:
        raise ValueError("table length %d != R %d" % (Rt, R))
    if q_rows.shape != (n, d) or rs_rows.shape != (n, C):
        raise ValueError("q_rows / rs_rows shape mismatch")
    return _rows_call(lib, q_rows, rs_rows, proj, k, v, req, B, T, Hq, Hkv, d, window, R, scale, temp_n0)


def _rows_call(lib, q_rows, rs_rows, proj, k, v, req, B, T, Hq, Hkv, d, window, R, scale, temp_n0=0):
    n = req.shape[0]
    Hp, C, _ = proj.shape
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    if n == 0:
        return o, lse
    rc = lib.oracle_attn_rows(q_rows.ctypes.data, rs_rows.ctypes.data, proj.ctypes.data, Hp, C,
                              k.ctypes.data, v.ctypes.data, req.ctypes.data, n,
                              B, T, Hq, Hkv, d, int(window), int(R), float(scale), int(temp_n0),
                              o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attn_rows rejected its arguments")
    return o, lse


def _tables(w, Hq: int, R: int) -> np.ndarray:
    """Distance tables as [Hp, C, R]: w [Hq, R] (rank 1, per head), [Hq, C, R] or [C, R] (shared)."""
    w = _f32(w)
    if w.ndim == 2 and w.shape == (Hq, R):
        return w.reshape(Hq, 1, R)
    if w.ndim == 3 and w.shape[0] in (1, Hq) and w.shape[2] == R:
        return w
    if w.ndim == 2 and w.shape[1] == R:  # one shared bank [C, R]
        return w.reshape(1, w.shape[0], R)
    raise ValueError("unsupported table shape %s for Hq=%d R=%d" % (w.shape, Hq, R))


def attn_prefill(q, k, v, r, w, window: int, R: int, scale: float, rows=None, temp_n0: int = 0):
    """Causal biased attention over whole sequences.

    q [B, T, Hq, d]; k, v [B, T, Hkv, d]; r [B, T, Hq] (rank 1) or [B, T, Hq, C];
    w [Hq, R] (rank 1, per head) or a bank [C, R] / [1, C, R] / [Hq, C, R].
    rows: None for every (b, h, i); else an [n, 3] array of (b, h, i).
    temp_n0: context-length temperature break point (see attn_rows); 0 = none.
    Returns (O [B, T, Hq, d], LSE [B, Hq, T]) in float64 for rows=None,
    else (o [n, d], lse [n]).
    """
    lib = _load()
    q = _f32(q)
    k = _f32(k)
    v = _f32(v)
    r = _f32(r)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != k.shape:
        raise ValueError("q %s, k %s, v %s do not fit [B,T,H,d]" % (q.shape, k.shape, v.shape))
    proj = _tables(w, Hq, R)
    C = proj.shape[1]
    if r.size != B * T * Hq * C:
        raise ValueError("r has %d values, expected B*T*Hq*C = %d" % (r.size, B * T * Hq * C))
    rs = r.reshape(B, T, Hq, C)
    if rows is None:
        b_i, t_i, h_i = np.meshgrid(np.arange(B), np.arange(T), np.arange(Hq), indexing="ij")
        req = np.stack([b_i.ravel(), h_i.ravel(), t_i.ravel()], axis=1).astype(np.int64)
    else:
        req = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        bad = (req < 0).any(axis=1) | (req[:, 0] >= B) | (req[:, 1] >= Hq) | (req[:, 2] >= T)
        if bad.any():
            raise ValueError("row request out of range: %s" % (req[bad][0].tolist(),))
    q_rows = np.ascontiguousarray(q[req[:, 0], req[:, 2], req[:, 1], :])
    rs_rows = np.ascontiguousarray(rs[req[:, 0], req[:, 2], req[:, 1], :])
    o, lse = _rows_call(lib, q_rows, rs_rows, proj, k, v, req, B, T, Hq, Hkv, d, window, R, scale, temp_n0)
    if rows is not None:
        return o, lse
    return o.reshape(B, T, Hq, d), lse.reshape(B, T, Hq).transpose(0, 2, 1).copy()


def attn_backward(q, k, v, r, w, dout, window: int, R: int, scale: float, temp_n0: int = 0):
    """Gradients of the prefill (relbias_oracle.c, oracle_attn_bwd, states the steps).

    Shapes as attn_prefill, plus dout [B, T, Hq, d] = dL/dO.  Returns a dict of fp64
    arrays: dq [B,T,Hq,d], dk and dv [B,T,Hkv,d], dr shaped like r, dw shaped like w.
    """
    lib = _load()
    q = _f32(q)
    k = _f32(k)
    v = _f32(v)
    r_in = _f32(r)
    w_in = _f32(w)
    dout = _f32(dout)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != k.shape or dout.shape != q.shape:
        raise ValueError("q %s, k %s, v %s, dout %s do not fit" % (q.shape, k.shape, v.shape, dout.shape))
    proj = np.ascontiguousarray(_tables(w_in, Hq, R))
    Hp, C, _ = proj.shape
    if r_in.size != B * T * Hq * C:
        raise ValueError("r has %d values, expected B*T*Hq*C = %d" % (r_in.size, B * T * Hq * C))
    rs = np.ascontiguousarray(r_in.reshape(B, T, Hq, C))
    dq = np.zeros((B, T, Hq, d))
    dk = np.zeros((B, T, Hkv, d))
    dv = np.zeros((B, T, Hkv, d))
    drs = np.zeros((B, T, Hq, C))
    dproj = np.zeros((Hp, C, max(R, 0)))
    rc = lib.oracle_attn_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, rs.ctypes.data, proj.ctypes.data, Hp, C,
                             dout.ctypes.data, B, T, Hq, Hkv, d, int(window), int(R), float(scale), int(temp_n0),
                             dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, drs.ctypes.data, dproj.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attn_bwd rejected its arguments")
    return {"dq": dq, "dk": dk, "dv": dv, "dr": drs.reshape(r_in.shape), "dw": dproj.reshape(w_in.shape)}


def attn_decode(q, k_cache, v_cache, r, w, window: int, R: int, scale: float, temp_n0: int = 0):
    """One new query per sequence at position n_ctx-1 against a cache of n_ctx rows
    that already holds the query's own key and value in its last row.

    q [B, Hq, d]; k_cache, v_cache [B, n_ctx, Hkv, d]; r [B, Hq] or [B, Hq, C].
    temp_n0: context-length temperature break point (see attn_rows); 0 = none.
    Returns (O [B, Hq, d], LSE [B, Hq]) in float64.
    """
    lib = _load()
    q = _f32(q)
    k = _f32(k_cache)
    v = _f32(v_cache)
    r = _f32(r)
    B, Hq, d = q.shape
    _, N, Hkv, _ = k.shape
    if k.shape != (B, N, Hkv, d) or v.shape != k.shape:
        raise ValueError("q %s, k %s, v %s do not fit a [B,n_ctx,Hkv,d] cache" % (q.shape, k.shape, v.shape))
    proj = _tables(w, Hq, R)
    C = proj.shape[1]
    if r.size != B * Hq * C:
        raise ValueError("r has %d values, expected B*Hq*C = %d" % (r.size, B * Hq * C))
    b_i, h_i = np.meshgrid(np.arange(B), np.arange(Hq), indexing="ij")
    req = np.stack([b_i.ravel(), h_i.ravel(), np.full(B * Hq, N - 1)], axis=1).astype(np.int64)
    o, lse = _rows_call(lib, q.reshape(B * Hq, d), r.reshape(B * Hq, C), proj, k, v, req,
                        B, N, Hq, Hkv, d, window, R, scale, temp_n0)
    return o.reshape(B, Hq, d), lse.reshape(B, Hq)


def bias_matrix(rs, proj, positions, R: int) -> np.ndarray:
    """The whole bias tensor (H, T, T) for tiny inputs, one entry at a time.

    Entry (h, i, j) is the token's curve (coefficients times the distance table or
    bank, step 2 of the essay's recipe) read at distance pos_i - pos_j (step 3),
    and zero when that distance is negative or at least R (step 4).
    rs [T, H, C]; proj [C, R] (one bank shared by every head) or [H, C, R] (a table
    per head); positions [T].  Pure-Python loops in fp64: for T of a few dozen only.
    """
    rs = np.asarray(rs, dtype=np.float64)
    proj = np.asarray(proj, dtype=np.float64)
    pos = [int(p) for p in np.asarray(positions).ravel()]
    T, H, C = rs.shape
    out = np.zeros((H, T, T), dtype=np.float64)
    for h in range(H):
        table = proj if proj.ndim == 2 else proj[h]
        for i in range(T):
            for j in range(T):
                dist = pos[i] - pos[j]
                if 0 <= dist < R:
                    out[h, i, j] = sum(rs[i, h, c] * table[c, dist] for c in range(C))
    return out
