"""fp64 CPU oracle of the pi-attention forward operator -- TEST INFRASTRUCTURE ONLY.

Only tests/, the package smoke check (__graft_entry__.smoke) and bench.py's CPU-baseline leg may
import this package.  The product path never does, and the oracle never touches the CUDA path:
they share no code.  The arithmetic lives in pi_oracle.c (plain loops in double, one query row at
a time, written from the definition; see that file's header for the formulas and the passages
they follow).  This module compiles it with gcc on first use and marshals numpy arrays.

`brute` (brute.py) is a second, independent checker of this oracle: a dense n x n masked
softmax with an additive bias matrix, built in numpy from set definitions.

Parity status of each function (what pins it against something other than itself):
  index_set / counts / index_table   pinned: the worked mask count of the "Sliding Window
                                     Attention" page (58 vs 136), reach by layer (4, 7, 10, 13),
                                     closed-form totals, brute-force set enumeration
  fwd_rows / fwd                     pinned: dense brute force and torch SDPA with the bias as
                                     attn_mask; closed forms of the gate (q = 0 or k = 0); the
                                     alpha -> 1 / alpha -> 0 limits (causal sliding-window attention
                                     and skip-only attention); rows sum to 1
  decode                             pinned: equals fwd_rows on the last row of the same sequence,
                                     which is pinned as above
  bwd (gradients of a loss through    pinned: central finite differences of fwd (itself pinned);
  out: dq, dk, dv, dw_g, db_g)        torch autograd through a dense formulation of the operator
  bidir=True (two-sided window and    pinned: dense brute force (masks from |i - j|), closed-form
  skips, every function above but     totals, torch SDPA with the bias, alpha -> 1 = two-sided
  decode)                             sliding-window attention, reversing the sequence maps the
                                     operator onto itself
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pi_oracle.c")
_SO = os.path.join(_HERE, "_pi_oracle.so")
_lock = threading.Lock()
_lib_handle = None


def build(force: bool = False) -> str:
    """Compile pi_oracle.c into an in-tree shared library (gcc -O2; no fast-math)."""
    with _lock:
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            tmp = _SO + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, _SO)
    return _SO


def bind(lib):
    """Declare the C signatures on a loaded copy of the oracle library and return it."""
    i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.oracle_index_set.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp]
    lib.oracle_index_set.restype = i64
    lib.oracle_index_set_ex.argtypes = [i64, i64, i64, i64, i64, i32, vp, vp, vp, vp]
    lib.oracle_index_set_ex.restype = i64
    lib.oracle_counts_ex.argtypes = [i64, i64, i64, i64, i32, vp, vp]
    lib.oracle_counts_ex.restype = None
    lib.oracle_index_table_ex.argtypes = [i64, i64, i64, i64, i32, i64, vp, vp]
    lib.oracle_index_table_ex.restype = None
    lib.oracle_fwd_rows_ex.argtypes = [vp, vp, vp, i32, vp, vp, i64, i64, i64, i64, i64, i64, i64, i32, vp, i64, vp, vp,
                                       vp, i32]
    lib.oracle_fwd_rows_ex.restype = None
    lib.oracle_counts.argtypes = [i64, i64, i64, i64, vp, vp]
    lib.oracle_counts.restype = None
    lib.oracle_index_table.argtypes = [i64, i64, i64, i64, i64, vp, vp]
    lib.oracle_index_table.restype = None
    lib.oracle_fwd_rows.argtypes = [vp, vp, vp, i32, vp, vp, i64, i64, i64, i64, i64, i64, i64, vp, i64, vp, vp, vp,
                                    i32]
    lib.oracle_fwd_rows.restype = None
    lib.oracle_decode.argtypes = [vp, vp, vp, i32, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, vp, i64, vp, vp, vp,
                                  i32]
    lib.oracle_decode.restype = None
    lib.oracle_bwd.argtypes = [vp, vp, vp, i32, vp, vp, i64, i64, i64, i64, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp,
                               i32]
    lib.oracle_bwd.restype = None
    return lib


def _lib():
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = bind(ctypes.CDLL(build()))
    return _lib_handle


def _threads(n):
    return int(n) if n else max(1, os.cpu_count() or 1)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1  # bf16 bit patterns
    raise TypeError(f"oracle inputs must be float32 or bf16 bits (uint16), got {a.dtype}")


def index_set(i: int, kwin: int, pi: int, S: int, n: int | None = None, bidir: bool = False):
    """(L(i) ascending, P(i) by increasing m) as int64 arrays.  bidir: two-sided window and skips in
    a sequence of n tokens (P lists i - m pi before i + m pi for each m)."""
    if bidir and n is None:
        raise ValueError("the bidirectional index rule needs the sequence length n")
    L = np.empty(2 * kwin + 1, dtype=np.int64)
    P = np.empty(max(2 * S, 1), dtype=np.int64)
    nL = np.zeros(1, dtype=np.int64)
    nP = np.zeros(1, dtype=np.int64)
    _lib().oracle_index_set_ex(i, i + 1 if n is None else n, kwin, pi, S, int(bidir), L.ctypes.data, nL.ctypes.data,
                               P.ctypes.data, nP.ctypes.data)
    return L[: nL[0]].copy(), P[: nP[0]].copy()


def counts(n: int, kwin: int, pi: int, S: int, bidir: bool = False):
    """(sum_i |L(i)|, sum_i |P(i)|) over i = 0..n-1."""
    a = np.zeros(1, dtype=np.int64)
    b = np.zeros(1, dtype=np.int64)
    _lib().oracle_counts_ex(n, kwin, pi, S, int(bidir), a.ctypes.data, b.ctypes.data)
    return int(a[0]), int(b[0])


def index_table(n: int, kwin: int, pi: int, S: int, width: int | None = None, bidir: bool = False):
    """counts [n, 2] int32 and idx [n, width] int32 (L ascending, then P by m, then -1)."""
    if width is None:
        width = 2 * kwin + 1 + 2 * S if bidir else kwin + 1 + S
    c = np.zeros((n, 2), dtype=np.int32)
    idx = np.zeros((n, width), dtype=np.int32)
    _lib().oracle_index_table_ex(n, kwin, pi, S, int(bidir), width, c.ctypes.data, idx.ctypes.data)
    return c, idx


def fwd_rows(q, k, v, w_g, b_g, kwin: int, pi: int, S: int, rows=None, nthreads: int | None = None,
             bidir: bool = False):
    """Oracle on selected query rows (bidir: two-sided window and skips).

    q, k, v: [B, H, n, d] float32 or bf16 bits (uint16).  w_g [H, d], b_g [H] float32.
    rows: flat indices (b*H + h)*n + i (default: all rows).
    Returns out [nrows, d], lse [nrows], rowsum [nrows] in float64."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    dt = _dtype_code(q)
    assert _dtype_code(k) == dt and _dtype_code(v) == dt
    B, H, n, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    w_g = np.ascontiguousarray(w_g, dtype=np.float32).reshape(H, d)
    b_g = np.ascontiguousarray(b_g, dtype=np.float32).reshape(H)
    if rows is None:
        rows = np.arange(B * H * n, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, d), dtype=np.float64)
    lse = np.zeros(rows.size, dtype=np.float64)
    rs = np.zeros(rows.size, dtype=np.float64)
    _lib().oracle_fwd_rows_ex(q.ctypes.data, k.ctypes.data, v.ctypes.data, dt, w_g.ctypes.data, b_g.ctypes.data, B,
                              H, n, d, kwin, pi, S, int(bidir), rows.ctypes.data, rows.size, out.ctypes.data,
                              lse.ctypes.data, rs.ctypes.data, _threads(nthreads))
    return out, lse, rs


def fwd(q, k, v, w_g, b_g, kwin: int, pi: int, S: int, nthreads: int | None = None, bidir: bool = False):
    """Oracle on every row: out [B, H, n, d], lse [B, H, n], rowsum [B, H, n] (float64)."""
    B, H, n, d = q.shape
    out, lse, rs = fwd_rows(q, k, v, w_g, b_g, kwin, pi, S, None, nthreads, bidir=bidir)
    return out.reshape(B, H, n, d), lse.reshape(B, H, n), rs.reshape(B, H, n)


def decode(q, kc, vc, w_g, b_g, kwin: int, pi: int, S: int, lengths=None, bh=None, nthreads: int | None = None):
    """Decode oracle.  q [B, H, d]; kc, vc [B, H, n_cache, d]; lengths int32 [B] or None.
    bh: list of b*H + h to evaluate (default all).  Returns out [nbh, d], lse [nbh], rowsum [nbh]."""
    q = np.ascontiguousarray(q)
    kc = np.ascontiguousarray(kc)
    vc = np.ascontiguousarray(vc)
    dt = _dtype_code(q)
    assert _dtype_code(kc) == dt and _dtype_code(vc) == dt
    B, H, d = q.shape
    n_cache = kc.shape[2]
    assert kc.shape == (B, H, n_cache, d) and vc.shape == kc.shape
    w_g = np.ascontiguousarray(w_g, dtype=np.float32).reshape(H, d)
    b_g = np.ascontiguousarray(b_g, dtype=np.float32).reshape(H)
    if bh is None:
        bh = np.arange(B * H, dtype=np.int64)
    bh = np.ascontiguousarray(bh, dtype=np.int64)
    lp = None
    if lengths is not None:
        lengths = np.ascontiguousarray(lengths, dtype=np.int32).reshape(B)
        lp = lengths.ctypes.data
    out = np.zeros((bh.size, d), dtype=np.float64)
    lse = np.zeros(bh.size, dtype=np.float64)
    rs = np.zeros(bh.size, dtype=np.float64)
    _lib().oracle_decode(q.ctypes.data, kc.ctypes.data, vc.ctypes.data, dt, w_g.ctypes.data, b_g.ctypes.data, lp, B, H,
                         n_cache, d, kwin, pi, S, bh.ctypes.data, bh.size, out.ctypes.data, lse.ctypes.data,
                         rs.ctypes.data, _threads(nthreads))
    return out, lse, rs


def bwd(q, k, v, w_g, b_g, dO, kwin: int, pi: int, S: int, bidir: bool = False, nthreads: int | None = None,
        return_terms: bool = False):
    """Gradients of a scalar loss through out, given dO = dLoss/dout [B, H, n, d].
    q, k, v as for fwd.  Returns dq, dk, dv [B, H, n, d], dw_g [H, d], db_g [H] (float64); with
    return_terms also terms [B, H, n, 3]: per row dz_i (its term in db_g), D_i = dO_i . out_i and
    sum_j p_j^2 (dO_i . v_j)^2."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    dt = _dtype_code(q)
    assert _dtype_code(k) == dt and _dtype_code(v) == dt
    B, H, n, d = q.shape
    w_g = np.ascontiguousarray(w_g, dtype=np.float32).reshape(H, d)
    b_g = np.ascontiguousarray(b_g, dtype=np.float32).reshape(H)
    dO = np.ascontiguousarray(dO, dtype=np.float64).reshape(B, H, n, d)
    dq, dk, dv = (np.zeros((B, H, n, d), dtype=np.float64) for _ in range(3))
    dw = np.zeros((H, d), dtype=np.float64)
    db = np.zeros(H, dtype=np.float64)
    terms = np.zeros((B, H, n, 3), dtype=np.float64) if return_terms else None
    _lib().oracle_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, dt, w_g.ctypes.data, b_g.ctypes.data, B, H, n, d,
                      kwin, pi, S, int(bidir), dO.ctypes.data, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data,
                      dw.ctypes.data, db.ctypes.data, None if terms is None else terms.ctypes.data, _threads(nthreads))
    if return_terms:
        return dq, dk, dv, dw, db, terms
    return dq, dk, dv, dw, db
