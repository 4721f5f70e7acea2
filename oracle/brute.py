"""Brute-force checker of the oracle -- TEST INFRASTRUCTURE ONLY.

A second, independent statement of the operator for tiny inputs: build the dense n x n additive
bias matrix and run textbook softmax attention with dense matrix products.  The "Sliding Window
Attention" glossary page (section "Wie das Fenster mit der Tiefe wächst") notes that the same
boolean mask can be handed to a library attention routine as its attention mask; this module is
that idea with the pi-attention pattern and gate:

  window mask  W[i, j] = 0 <= i - j <= k                        (dense comparison of positions)
  skip mask    C[i, j] = (i - j) in {pi, 2 pi, ..., S pi},  skip = C and not W
  bidirectional: W[i, j] = |i - j| <= k,  C[i, j] = |i - j| in {pi, ..., S pi}
               (set difference: a skip key inside the window stays a window key)
  bias         log(alpha_i) on W, log(1 - alpha_i) on skip, -inf elsewhere,
               alpha_i = sigmoid(q_i . w_g + b_g)  (log-sigmoid from scipy)
  attention    softmax(tau * Q K^T + bias) V,  lse = logsumexp(tau * Q K^T + bias)

None of this shares code or formulas' layout with pi_oracle.c (per-row loops over index lists).
"""
from __future__ import annotations

import numpy as np
from scipy.special import log_expit, logsumexp


def masks(n: int, kwin: int, pi: int, S: int, bidir: bool = False):
    """Dense boolean window and skip masks [n, n] (query row, key column)."""
    pos = np.arange(n)
    off = pos[:, None] - pos[None, :]
    if bidir:
        off = np.abs(off)
    W = (off >= 0) & (off <= kwin)
    C = np.zeros((n, n), dtype=bool)
    for m in range(1, S + 1):
        C |= off == m * pi
    return W, C & ~W


def widen(a: np.ndarray) -> np.ndarray:
    """Stored inputs as float64 (bf16 bit patterns are widened exactly)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def attention(q, k, v, w_g, b_g, kwin: int, pi: int, S: int, bidir: bool = False):
    """q, k, v [B, H, n, d] (float32 or bf16 bits) -> out [B, H, n, d], lse [B, H, n], bias [B, H, n, n]."""
    q, k, v = widen(q), widen(k), widen(v)
    B, H, n, d = q.shape
    w_g = np.asarray(w_g, dtype=np.float64).reshape(H, d)
    b_g = np.asarray(b_g, dtype=np.float64).reshape(H)
    W, P = masks(n, kwin, pi, S, bidir)
    z = np.einsum("bhnd,hd->bhn", q, w_g) + b_g[None, :, None]
    log_a = log_expit(z)
    log_1ma = log_expit(-z)
    bias = np.full((B, H, n, n), -np.inf)
    bias = np.where(W[None, None], log_a[..., None], bias)
    bias = np.where(P[None, None], log_1ma[..., None], bias)
    scores = np.einsum("bhid,bhjd->bhij", q, k) / np.sqrt(d) + bias
    lse = logsumexp(scores, axis=-1)
    p = np.exp(scores - lse[..., None])
    out = np.einsum("bhij,bhjd->bhid", p, v)
    return out, lse, bias
