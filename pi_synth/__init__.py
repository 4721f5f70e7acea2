"""Seeded synthetic inputs for the pi-attention operator, its tests and its bench.

This module draws numbers and nothing else: it holds none of the operator's arithmetic, so
the fp64 oracle and the CUDA path can both read what it writes.  The generator itself is the
C file beside this one (Philox4x32-10 + Box-Muller, see its header); this file compiles it on
first use, wraps it with ctypes and holds the workload recipes.

Workloads (the shapes and value distributions the method is measured on):

  tiny_f32     fp32, B=1 H=2 n=256 d=32, window k=8, period pi=16, S=2 skips;
               q,k,v ~ N(0,1); w_g ~ N(0,1/d); b_g = 0
  bf16_n4k     bf16, B=1 H=8 n=4096 d=64, k=128, pi=64, S=4;
               q,k,v ~ N(0,1); w_g ~ N(0,1/d); b_g ~ N(0,0.5)
  bf16_n32k    bf16, B=2 H=16 n=32768 d=128, k=256, pi=256, S=8;
               q,k,v ~ N(0,1), every key row j with j % 256 == 0 scaled by 4 (K only);
               w_g ~ N(0,1/d); b_g = 0
  bf16_n128k   bf16, B=1 H=32 n=131072 d=128, k=512, pi=1024, S=16;
               q,k,v ~ N(0,1); w_g ~ N(0,1/d); b_g = 0
  decode_bf16  bf16 decode, B=64 H=32, cache of 65536 tokens, d=128, k=1024, pi=2048, S=31;
               q,k,v ~ N(0,1); w_g ~ N(0,1/d); b_g = 0

The second argument of N(., .) is the variance.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pi_synth.c")
_SO = os.path.join(_HERE, "_pi_synth.so")
_lock = threading.Lock()
_lib_handle = None

# stream ids: one independent Philox stream per tensor of a workload
STREAM_Q, STREAM_K, STREAM_V, STREAM_WG, STREAM_BG = 1, 2, 3, 4, 5
STREAM_DQ, STREAM_DK, STREAM_DV, STREAM_DWG, STREAM_DBG = 11, 12, 13, 14, 15
STREAM_DO = 6  # the loss gradient of the backward workloads


def build(force: bool = False) -> str:
    """Compile the generator into an in-tree shared library (gcc, -O2, pthreads)."""
    with _lock:
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            tmp = _SO + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, _SO)
    return _SO


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build())
        u64, u32, dbl, vp, i32 = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        lib.pi_synth_fill.argtypes = [vp, i32, u64, u64, u64, u32, dbl, dbl, u64, u64, u64, dbl, i32]
        lib.pi_synth_fill.restype = None
        lib.pi_synth_fill_rows.argtypes = [vp, i32, vp, u64, u64, u64, u32, dbl, dbl, u64, u64, dbl, i32]
        lib.pi_synth_fill_rows.restype = None
        lib.pi_synth_philox.argtypes = [vp, vp, vp]
        lib.pi_synth_philox.restype = None
        _lib_handle = lib
    return _lib_handle


def threads() -> int:
    return max(1, os.cpu_count() or 1)


def philox4x32_10(ctr, key):
    """The raw Philox4x32-10 block function (for its known-answer test)."""
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    _lib().pi_synth_philox(c.ctypes.data, k.ctypes.data, o.ctypes.data)
    return o


def normal(shape, *, seed: int, stream: int, std: float = 1.0, mean: float = 0.0, dtype: str = "bf16",
           scale_every: int = 0, scale_factor: float = 1.0) -> np.ndarray:
    """Tensor of the given shape, element e = mean + std * z_e (z from the (seed, stream) stream).

    dtype "bf16" returns the bf16 bit patterns as uint16; "f32" returns float32.
    scale_every > 0 scales every row (last axis) whose index along the second-to-last axis is a
    multiple of scale_every by scale_factor, before rounding.
    """
    shape = tuple(int(s) for s in shape)
    count = int(np.prod(shape)) if shape else 1
    is_bf16 = dtype == "bf16"
    out = np.empty(shape, dtype=np.uint16 if is_bf16 else np.float32)
    row_len = shape[-1] if len(shape) >= 1 else 1
    seq_rows = shape[-2] if len(shape) >= 2 else 1
    if count:
        _lib().pi_synth_fill(out.ctypes.data, int(is_bf16), 0, count, seed, stream, mean, std, row_len, seq_rows,
                             scale_every, scale_factor, threads())
    return out


def rows(shape, flat_rows, *, seed: int, stream: int, std: float = 1.0, mean: float = 0.0,
         dtype: str = "bf16", scale_every: int = 0, scale_factor: float = 1.0) -> np.ndarray:
    """Selected rows (flat row indices over all but the last axis) of the tensor `normal(shape, ...)`
    would return, as an array [len(flat_rows), shape[-1]] holding the identical values."""
    shape = tuple(int(s) for s in shape)
    fr = np.ascontiguousarray(np.asarray(flat_rows, dtype=np.int64))
    is_bf16 = dtype == "bf16"
    out = np.empty((fr.size, shape[-1]), dtype=np.uint16 if is_bf16 else np.float32)
    if fr.size:
        _lib().pi_synth_fill_rows(out.ctypes.data, int(is_bf16), fr.ctypes.data, fr.size, shape[-1], seed, stream,
                                  mean, std, shape[-2] if len(shape) >= 2 else 1, scale_every, scale_factor, threads())
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) and return the bit patterns; finite inputs only."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill", "decode" or "backward" (gradients through a prefill)
    dtype: str           # "f32" or "bf16": storage type of q, k, v, out
    B: int
    H: int
    n: int               # sequence length (prefill) or cache length (decode)
    d: int
    k: int               # window: the token itself plus the k tokens before it
    pi: int              # skip period
    S: int               # skips i - m*pi for m = 1..S
    bg_std: float = 0.0  # std of b_g (0 means b_g = 0)
    k_scale_every: int = 0
    k_scale_factor: float = 1.0
    sampled_rows: int = 0  # > 0: parity on this many sampled query rows (plus boundary rows)
    bidir: bool = False    # the bidirectional index rule (two-sided window, skips i +- m*pi)

    @property
    def wg_std(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> dict:
        d = {"workload": self.name, "kind": self.kind, "dtype": self.dtype, "B": self.B, "H": self.H,
             "n": self.n, "d": self.d, "k": self.k, "pi": self.pi, "S": self.S}
        if self.bidir:
            d["bidir"] = True
        return d


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_f32", "prefill", "f32", 1, 2, 256, 32, 8, 16, 2),
        Workload("bf16_n4k", "prefill", "bf16", 1, 8, 4096, 64, 128, 64, 4, bg_std=math.sqrt(0.5)),
        Workload("bf16_n32k", "prefill", "bf16", 2, 16, 32768, 128, 256, 256, 8, k_scale_every=256,
                 k_scale_factor=4.0),
        Workload("bf16_n128k", "prefill", "bf16", 1, 32, 131072, 128, 512, 1024, 16, sampled_rows=4096),
        Workload("decode_bf16", "decode", "bf16", 64, 32, 65536, 128, 1024, 2048, 31),
        # the bf16_n4k recipe under the bidirectional rule (the pages' non-causal variant)
        Workload("bf16_n4k_bidir", "prefill", "bf16", 1, 8, 4096, 64, 128, 64, 4, bg_std=math.sqrt(0.5), bidir=True),
        # the backward (gradients through out) of the bf16_n4k recipe; dO ~ N(0, 1)
        Workload("bf16_n4k_bwd", "backward", "bf16", 1, 8, 4096, 64, 128, 64, 4, bg_std=math.sqrt(0.5)),
        # the backward of the bf16_n32k recipe: a long context, where the tensor-core backward takes
        # the split (residue-class) passes
        Workload("bf16_n32k_bwd", "backward", "bf16", 2, 16, 32768, 128, 256, 256, 8, k_scale_every=256,
                 k_scale_factor=4.0),
        # the decode step's launch shape (64 x 32 (b, h), one CTA each, k = 1024, S = 31) over a
        # 4096-row cache (pi = 128: skips m = 9..31 lie in the cache): a case small enough for
        # Nsight Compute
        Workload("decode_bf16_c4k", "decode", "bf16", 64, 32, 4096, 128, 1024, 128, 31),
        # the bf16_n128k recipe with 4 heads instead of 32: the same per-(b, h) geometry and launch
        # shape per head (inputs 384 MB, above the L2), small enough for Nsight Compute
        Workload("bf16_n128k_h4", "prefill", "bf16", 1, 4, 131072, 128, 512, 1024, 16, sampled_rows=512),
    ]
}


def gate_params(w: Workload, seed: int = 0, decode: bool = False):
    """w_g [H, d] ~ N(0, 1/d) and b_g [H] (fp32), per the workload recipe."""
    s_wg, s_bg = (STREAM_DWG, STREAM_DBG) if decode else (STREAM_WG, STREAM_BG)
    w_g = normal((w.H, w.d), seed=seed, stream=s_wg, std=w.wg_std, dtype="f32")
    if w.bg_std > 0:
        b_g = normal((w.H,), seed=seed, stream=s_bg, std=w.bg_std, dtype="f32")
    else:
        b_g = np.zeros((w.H,), dtype=np.float32)
    return w_g, b_g


def prefill_inputs(w: Workload, seed: int = 0) -> dict:
    """q, k, v [B, H, n, d] in the storage dtype (bf16 as uint16 bits), w_g [H, d], b_g [H]."""
    shp = (w.B, w.H, w.n, w.d)
    q = normal(shp, seed=seed, stream=STREAM_Q, dtype=w.dtype)
    k = normal(shp, seed=seed, stream=STREAM_K, dtype=w.dtype, scale_every=w.k_scale_every,
               scale_factor=w.k_scale_factor)
    v = normal(shp, seed=seed, stream=STREAM_V, dtype=w.dtype)
    w_g, b_g = gate_params(w, seed)
    return {"q": q, "k": k, "v": v, "w_g": w_g, "b_g": b_g}


def prefill_rows(w: Workload, s0: int, s1: int, seed: int = 0) -> dict:
    """Rows [s0, s1) of every (b, h) sequence of prefill_inputs(w, seed): q, k, v [B, H, s1 - s0, d]
    holding the identical values (each row regenerated alone), and the full w_g, b_g."""
    s0, s1 = max(0, int(s0)), min(w.n, int(s1))
    shp = (w.B, w.H, w.n, w.d)
    rows_ = (np.arange(w.B * w.H, dtype=np.int64)[:, None] * w.n + np.arange(s0, s1, dtype=np.int64)[None, :]).reshape(-1)
    out = {}
    for name, stream in (("q", STREAM_Q), ("k", STREAM_K), ("v", STREAM_V)):
        extra = dict(scale_every=w.k_scale_every, scale_factor=w.k_scale_factor) if name == "k" else {}
        out[name] = rows(shp, rows_, seed=seed, stream=stream, dtype=w.dtype, **extra).reshape(w.B, w.H, s1 - s0, w.d)
    out["w_g"], out["b_g"] = gate_params(w, seed)
    return out


def backward_inputs(w: Workload, seed: int = 0) -> dict:
    """prefill_inputs plus dO [B, H, n, d] ~ N(0, 1) in the storage dtype (the loss gradient)."""
    inp = prefill_inputs(w, seed)
    inp["dO"] = normal((w.B, w.H, w.n, w.d), seed=seed, stream=STREAM_DO, dtype=w.dtype)
    return inp


def decode_positions(n_cache: int, k: int, pi: int, S: int, length: int | None = None) -> np.ndarray:
    """Cache rows of the decode workload that hold generated values.

    The workload's storage plan: the last k+1 rows before and at position length-1, and every
    row length-1 - m*pi for m = 1..S.  It is a superset of what a query may read (it makes no
    de-duplication decision); all other rows stay NaN, so a stray read shows.  It is data
    placement, not the operator: the oracle and the kernels each apply the index rule themselves."""
    L = n_cache if length is None else length
    i = L - 1
    win = np.arange(max(0, i - k), i + 1, dtype=np.int64)
    sk = i - np.arange(1, S + 1, dtype=np.int64) * pi
    sk = sk[sk >= 0]
    return np.unique(np.concatenate([win, sk]))


def decode_inputs(w: Workload, seed: int = 0) -> dict:
    """Decode workload: q [B,H,d], plus the cache rows that hold data.

    Returns q, w_g, b_g, `pos` (the cache row positions that hold generated values, same for every
    (b, h)), and kc, vc [B, H, len(pos), d]: row r of (b, h) is cache row pos[r] of the full cache
    tensor [B, H, n_cache, d].  Every other cache row is NaN (all bits set)."""
    pos = decode_positions(w.n, w.k, w.pi, w.S)
    shp_c = (w.B, w.H, w.n, w.d)
    bh = np.arange(w.B * w.H, dtype=np.int64)
    flat = (bh[:, None] * w.n + pos[None, :]).reshape(-1)
    kc = rows(shp_c, flat, seed=seed, stream=STREAM_DK, dtype=w.dtype).reshape(w.B, w.H, pos.size, w.d)
    vc = rows(shp_c, flat, seed=seed, stream=STREAM_DV, dtype=w.dtype).reshape(w.B, w.H, pos.size, w.d)
    q = normal((w.B, w.H, w.d), seed=seed, stream=STREAM_DQ, dtype=w.dtype)
    w_g, b_g = gate_params(w, seed, decode=True)
    return {"q": q, "kc": kc, "vc": vc, "pos": pos, "w_g": w_g, "b_g": b_g}


NAN_BITS_BF16 = np.uint16(0xFFFF)
NAN_BITS_F32 = np.uint32(0xFFFFFFFF)
