"""Python binding of libpiattn (include/pi_attn.h): argument marshalling only.

Every step of the operator runs in the CUDA library; this module converts torch CUDA tensors to
device pointers, passes the caller's current stream and turns status codes into exceptions.
There is no CPU fallback: without the built library (or without a GPU) the calls raise.

    import periodic_sparse_attention_b200 as pia
    out, lse = pia.pi_attn_fwd(q, k, v, w_g, b_g, k_win=128, pi=64, S=4)
    out, lse = pia.pi_attn_decode(q, kcache, vcache, w_g, b_g, k_win=1024, pi=2048, S=31)
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpiattn.so")

PI_ATTN_OK, PI_ATTN_EINVAL, PI_ATTN_EUNSUPPORTED, PI_ATTN_ECUDA, PI_ATTN_EDEVICE = range(5)
PI_ATTN_F32, PI_ATTN_BF16 = 0, 1
PATHS = {"auto": 0, "simt": 1, "tc": 2, "tc_fused": 3, "tc_split": 4}

# (name, restype, argtypes) of every symbol include/pi_attn.h declares
_vp, _i32, _cstr = ctypes.c_void_p, ctypes.c_int, ctypes.c_char_p
SIGNATURES = {
    # 7 tensor pointers, B H n d k_win pi S, dtype, stream
    "pi_attn_fwd": (_i32, [_vp] * 7 + [_i32] * 8 + [_vp]),
    # ... as above plus the path selector
    "pi_attn_fwd_ex": (_i32, [_vp] * 7 + [_i32] * 9 + [_vp]),
    # 7 tensor pointers, B H n_q n_kv, row0 kv0 (int64), d k_win pi S, dtype, stream
    "pi_attn_fwd_shard": (_i32, [_vp] * 7 + [_i32] * 4 + [ctypes.c_longlong] * 2 + [_i32] * 5 + [_vp]),
    # ... plus workspace pointer and bytes before the stream
    "pi_attn_fwd_shard_ws": (_i32, [_vp] * 7 + [_i32] * 4 + [ctypes.c_longlong] * 2 + [_i32] * 5 +
                             [_vp, ctypes.c_longlong, _vp]),
    # B H n_q, row0 kv0 (int64), d k_win pi S
    "pi_attn_fwd_shard_scratch_bytes": (ctypes.c_longlong, [_i32] * 3 + [ctypes.c_longlong] * 2 + [_i32] * 4),
    # as pi_attn_fwd_ex, bidirectional index rule
    "pi_attn_fwd_bidir": (_i32, [_vp] * 7 + [_i32] * 9 + [_vp]),
    # ... plus workspace pointer and its size in bytes
    "pi_attn_fwd_ws": (_i32, [_vp] * 7 + [_i32] * 9 + [_vp, ctypes.c_longlong, _vp]),
    # 7 pointers (q k v host, w_g b_g device, out lse host), B H n d k_win pi S, dtype, path, chunk_heads,
    # device workspace, its bytes, stream
    "pi_attn_fwd_host": (_i32, [_vp] * 7 + [_i32] * 10 + [_vp, ctypes.c_longlong, _vp]),
    "pi_attn_fwd_host_workspace_bytes": (ctypes.c_longlong, [_i32] * 6),
    # B H n d k_win pi S, dtype, path, out: launches, scratch bytes
    "pi_attn_fwd_plan": (_i32, [_i32] * 9 + [_vp, _vp]),
    # 8 pointers (q kcache vcache w_g b_g cache_len out lse), B H n_cache d k_win pi S, dtype, stream
    "pi_attn_decode": (_i32, [_vp] * 8 + [_i32] * 8 + [_vp]),
    # as pi_attn_decode; no allocation (fixed 4 MiB device scratch inside the library)
    "pi_attn_decode_noalloc": (_i32, [_vp] * 8 + [_i32] * 8 + [_vp]),
    "pi_attn_debug_index_sets": (_i32, [_i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp]),
    "pi_attn_debug_index_sets_bidir": (_i32, [_i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp]),
    # q k v w_g b_g dout dq dk dv dw_g db_g, B H n d k_win pi S dtype bidir, workspace, bytes, stream
    "pi_attn_bwd": (_i32, [_vp] * 11 + [_i32] * 9 + [_vp, ctypes.c_longlong, _vp]),
    "pi_attn_bwd_workspace_bytes": (ctypes.c_longlong, [_i32, _i32, _i32, _i32]),
    # as pi_attn_bwd plus the kernel choice before the workspace
    "pi_attn_bwd_ex": (_i32, [_vp] * 11 + [_i32] * 10 + [_vp, ctypes.c_longlong, _vp]),
    "pi_attn_bwd_workspace_bytes_ex": (ctypes.c_longlong, [_i32] * 6),
    # as pi_attn_bwd_ex (q k v dout dq dk dv on the host) plus chunk_heads before the workspace
    "pi_attn_bwd_host": (_i32, [_vp] * 11 + [_i32] * 11 + [_vp, ctypes.c_longlong, _vp]),
    "pi_attn_bwd_host_workspace_bytes": (ctypes.c_longlong, [_i32] * 7),
    # as pi_attn_decode, capacity in place of n_cache
    "pi_attn_decode_ring": (_i32, [_vp] * 8 + [_i32] * 8 + [_vp]),
    # kcache vcache k_new v_new cache_len, B H capacity d dtype ring, stream
    "pi_attn_cache_append": (_i32, [_vp] * 5 + [_i32] * 6 + [_vp]),
    "pi_attn_check": (_i32, [_vp]),
    "pi_attn_status_string": (_cstr, [_i32]),
    "pi_attn_last_error": (_cstr, []),
    "pi_attn_version": (_i32, []),
}

_lib = None


class PiAttnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_status_name(status)}: {msg}")
        self.status = status


def _status_name(s):
    return ["PI_ATTN_OK", "PI_ATTN_EINVAL", "PI_ATTN_EUNSUPPORTED", "PI_ATTN_ECUDA", "PI_ATTN_EDEVICE"][s] \
        if 0 <= s < 5 else f"status {s}"


def load(path: str = LIB_PATH):
    """Load libpiattn.so (built by `build.build()`), declaring every exported signature."""
    global _lib
    if _lib is None or path != LIB_PATH:
        if not os.path.exists(path):
            raise ImportError(f"libpiattn.so not built at {path}; run python -m periodic_sparse_attention_b200.build")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        if path != LIB_PATH:
            return lib
        _lib = lib
    return _lib


def _raise(st: int):
    if st != PI_ATTN_OK:
        raise PiAttnError(st, load().pi_attn_last_error().decode())


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return PI_ATTN_F32
    if t.dtype == torch.bfloat16:
        return PI_ATTN_BF16
    raise TypeError(f"pi-attention tensors must be float32 or bfloat16, got {t.dtype}")


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("pi-attention tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("pi-attention tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_plans = {}


def pi_attn_fwd(q, k, v, w_g, b_g, k_win: int, pi: int, S: int, out=None, lse=None, *, path: str = "auto",
                stream=None, want_lse: bool = True, workspace=None, bidir: bool = False):
    """Prefill forward on torch CUDA tensors q, k, v [B, H, n, d] (fp32 or bf16), w_g [H, d] and
    b_g [H] (fp32).  Allocates out (q's dtype) and lse (fp32 [B, H, n]) when not given, and the
    split path's workspace (a uint8 tensor of pi_attn_fwd_plan's scratch bytes) from torch's
    caching allocator when not given.  bidir: the bidirectional rule (pi_attn_fwd_bidir)."""
    import torch
    B, H, n, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    dt = _dtype_code(q)
    if bidir:
        st = load().pi_attn_fwd_bidir(_ptr(q), _ptr(k), _ptr(v), _ptr(w_g), _ptr(b_g), _ptr(out), _ptr(lse), B, H, n,
                                      d, k_win, pi, S, dt, PATHS[path], _stream(stream))
        _raise(st)
        return out, lse
    key = (B, H, n, d, k_win, pi, S, dt, path)
    scratch = _plans.get(key)
    if scratch is None:
        scratch = pi_attn_fwd_plan(B, H, n, d, k_win, pi, S, "bf16" if dt == PI_ATTN_BF16 else "f32", path)[1]
        _plans[key] = scratch
    if workspace is None and scratch > 0:
        workspace = torch.empty(scratch, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().pi_attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(w_g), _ptr(b_g), _ptr(out), _ptr(lse), B, H, n, d,
                               k_win, pi, S, dt, PATHS[path], _ptr(workspace), ws_bytes, _stream(stream))
    _raise(st)
    return out, lse


def pi_attn_fwd_shard(q, k, v, w_g, b_g, k_win: int, pi: int, S: int, row0: int, kv0: int, out=None, lse=None, *,
                      stream=None, want_lse: bool = True, workspace=None):
    """One shard of a causal prefill: q [B, H, n_q, d] holds sequence rows row0 .., k and v
    [B, H, n_kv, d] hold sequence rows kv0 .. (the halo, then the shard's rows).  bf16, d in
    {64, 128}.  Allocates out and lse when not given, and the split path's workspace (a uint8
    tensor of pi_attn_fwd_shard_scratch_bytes) from torch's caching allocator when not given."""
    import torch
    B, H, n_q, d = q.shape
    n_kv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, n_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = load().pi_attn_fwd_shard_scratch_bytes(B, H, n_q, row0, kv0, d, k_win, pi, S)
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().pi_attn_fwd_shard_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(w_g), _ptr(b_g), _ptr(out), _ptr(lse), B, H, n_q,
                                     n_kv, row0, kv0, d, k_win, pi, S, _dtype_code(q), _ptr(workspace), ws_bytes,
                                     _stream(stream))
    _raise(st)
    return out, lse


def _hptr(t):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("pi_attn_fwd_host takes q, k, v, out and lse in host memory")
    if not t.is_contiguous():
        raise ValueError("pi-attention tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def pi_attn_fwd_host_workspace_bytes(B: int, H: int, n: int, d: int, dtype: str = "bf16", chunk_heads: int = 0):
    return load().pi_attn_fwd_host_workspace_bytes(B, H, n, d, PI_ATTN_BF16 if dtype == "bf16" else PI_ATTN_F32,
                                                   chunk_heads)


def pi_attn_fwd_host(q, k, v, w_g, b_g, k_win: int, pi: int, S: int, out=None, lse=None, *, path: str = "auto",
                     chunk_heads: int = 0, workspace=None, stream=None, want_lse: bool = True):
    """Prefill forward with q, k, v, out and lse in host memory (torch CPU tensors; pinned for the
    copies to overlap), w_g and b_g on the device: pi_attn_fwd_host, a pipeline of chunks of
    chunk_heads heads.  Allocates out and lse (pinned) when not given and the device workspace
    from torch's caching allocator when not given.  The results are on the host once the stream
    has been synchronized (this function does not synchronize)."""
    import torch
    B, H, n, d = q.shape
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    if lse is None and want_lse:
        lse = torch.empty((B, H, n), dtype=torch.float32).pin_memory()
    dt = _dtype_code(q)
    if workspace is None:
        nbytes = pi_attn_fwd_host_workspace_bytes(B, H, n, d, "bf16" if dt == PI_ATTN_BF16 else "f32", chunk_heads)
        if nbytes < 0:
            raise ValueError(f"invalid sizes for pi_attn_fwd_host: {tuple(q.shape)}, chunk_heads={chunk_heads}")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=w_g.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load().pi_attn_fwd_host(_hptr(q), _hptr(k), _hptr(v), _ptr(w_g), _ptr(b_g), _hptr(out), _hptr(lse), B, H, n,
                                 d, k_win, pi, S, dt, PATHS[path], chunk_heads, _ptr(workspace), ws_bytes,
                                 _stream(stream))
    _raise(st)
    return out, lse


def pi_attn_bwd_host(q, k, v, w_g, b_g, dout, k_win: int, pi: int, S: int, *, bidir: bool = False, grads=None,
                     path: str = "auto", chunk_heads: int = 0, workspace=None, stream=None):
    """Gradients with q, k, v, dout (torch CPU tensors; pinned for the copies to overlap) and dq, dk,
    dv (fp32, pinned, allocated when grads is None) in host memory; w_g, b_g and dw_g, db_g on the
    device: pi_attn_bwd_host, a pipeline of chunks of chunk_heads heads.  Returns (dq, dk, dv, dw_g,
    db_g); the host gradients are complete once the stream has been synchronized."""
    import torch
    B, H, n, d = q.shape
    if grads is None:
        grads = tuple(torch.empty((B, H, n, d), dtype=torch.float32).pin_memory() for _ in range(3)) + (
            torch.empty((H, d), dtype=torch.float32, device=w_g.device),
            torch.empty((H,), dtype=torch.float32, device=w_g.device))
    dq, dk, dv, dw, db = grads
    dt = _dtype_code(q)
    if workspace is None:
        nbytes = load().pi_attn_bwd_host_workspace_bytes(B, H, n, d, dt, BWD_PATHS[path], chunk_heads)
        if nbytes < 0:
            raise ValueError(f"invalid sizes for pi_attn_bwd_host: {tuple(q.shape)}, chunk_heads={chunk_heads}")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=w_g.device)
    st = load().pi_attn_bwd_host(_hptr(q), _hptr(k), _hptr(v), _ptr(w_g), _ptr(b_g), _hptr(dout), _hptr(dq),
                                 _hptr(dk), _hptr(dv), _ptr(dw), _ptr(db), B, H, n, d, k_win, pi, S, dt, int(bidir),
                                 BWD_PATHS[path], chunk_heads, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st)
    return dq, dk, dv, dw, db


def pi_attn_fwd_plan(B: int, H: int, n: int, d: int, k_win: int, pi: int, S: int, dtype: str = "bf16",
                     path: str = "auto"):
    """(kernel launches, scratch bytes) a pi_attn_fwd_ex call would use, without launching."""
    launches = ctypes.c_int(0)
    scratch = ctypes.c_longlong(0)
    st = load().pi_attn_fwd_plan(B, H, n, d, k_win, pi, S, PI_ATTN_BF16 if dtype == "bf16" else PI_ATTN_F32,
                                 PATHS[path], ctypes.byref(launches), ctypes.byref(scratch))
    _raise(st)
    return launches.value, scratch.value


def pi_attn_decode(q, kcache, vcache, w_g, b_g, k_win: int, pi: int, S: int, cache_len=None, out=None, lse=None, *,
                   stream=None, want_lse: bool = True):
    """Decode step: q [B, H, d], caches [B, H, n_cache, d], optional cache_len int32 [B] (device)."""
    import torch
    B, H, d = q.shape
    n_cache = kcache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = load().pi_attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(w_g), _ptr(b_g), _ptr(cache_len), _ptr(out),
                               _ptr(lse), B, H, n_cache, d, k_win, pi, S, _dtype_code(q), _stream(stream))
    _raise(st)
    return out, lse


def pi_attn_decode_noalloc(q, kcache, vcache, w_g, b_g, k_win: int, pi: int, S: int, cache_len=None, out=None,
                           lse=None, *, stream=None, want_lse: bool = True):
    """pi_attn_decode without any device allocation inside the call (its workspace is a fixed
    4 MiB array inside the library); out and lse are allocated here when not given."""
    import torch
    B, H, d = q.shape
    n_cache = kcache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = load().pi_attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(w_g), _ptr(b_g), _ptr(cache_len),
                                       _ptr(out), _ptr(lse), B, H, n_cache, d, k_win, pi, S, _dtype_code(q),
                                       _stream(stream))
    _raise(st)
    return out, lse


def pi_attn_debug_index_sets(n: int, k_win: int, pi: int, S: int, width: int | None = None, device="cuda",
                             stream=None, bidir: bool = False):
    """Index sets as the kernels enumerate them: counts [n, 2] and idx [n, width] int32 tensors."""
    import torch
    if width is None:
        width = 2 * k_win + 1 + 2 * S if bidir else k_win + 1 + S
    counts = torch.empty((n, 2), dtype=torch.int32, device=device)
    idx = torch.empty((n, width), dtype=torch.int32, device=device)
    fn = load().pi_attn_debug_index_sets_bidir if bidir else load().pi_attn_debug_index_sets
    st = fn(n, k_win, pi, S, _ptr(counts), _ptr(idx), width, _stream(stream))
    _raise(st)
    return counts, idx


BWD_PATHS = {"auto": 0, "simt": 1, "tc": 2, "tc_fused": 3, "tc_split": 4}


def pi_attn_bwd(q, k, v, w_g, b_g, dout, k_win: int, pi: int, S: int, *, bidir: bool = False, grads=None,
                workspace=None, stream=None, path: str = "simt"):
    """Gradients of a loss through out: (dq, dk, dv, dw_g, db_g), fp32 tensors.  q, k, v, dout
    [B, H, n, d] in one dtype (fp32 or bf16); w_g [H, d], b_g [H] fp32.  grads: a tuple of the five
    output tensors to write into (allocated when None); workspace from torch's caching allocator
    when None.  path: "simt" (pi_attn_bwd, fp32 throughout), "tc_fused" or "tc_split" (the
    tensor-core passes in one sweep, or split into a residue-class skip pass and a window pass),
    "tc" (the tensor cores, fused or split by shape) or "auto" (pi_attn_bwd_ex)."""
    import torch
    B, H, n, d = q.shape
    dev = q.device
    if grads is None:
        grads = (torch.empty((B, H, n, d), dtype=torch.float32, device=dev),
                 torch.empty((B, H, n, d), dtype=torch.float32, device=dev),
                 torch.empty((B, H, n, d), dtype=torch.float32, device=dev),
                 torch.empty((H, d), dtype=torch.float32, device=dev),
                 torch.empty((H,), dtype=torch.float32, device=dev))
    lib = load()
    dt, pc = _dtype_code(q), BWD_PATHS[path]
    if workspace is None:
        workspace = torch.empty(lib.pi_attn_bwd_workspace_bytes_ex(B, H, n, d, dt, pc), dtype=torch.uint8, device=dev)
    dq, dk, dv, dw, db = grads
    st = lib.pi_attn_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(w_g), _ptr(b_g), _ptr(dout), _ptr(dq), _ptr(dk),
                            _ptr(dv), _ptr(dw), _ptr(db), B, H, n, d, k_win, pi, S, dt, int(bidir), pc,
                            _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st)
    return dq, dk, dv, dw, db


def pi_attn_decode_ring(q, kcache, vcache, w_g, b_g, cache_len, k_win: int, pi: int, S: int, out=None, lse=None, *,
                        stream=None, want_lse: bool = True):
    """Decode over a ring cache: q [B, H, d]; caches [B, H, capacity, d] with position j in slot
    j mod capacity; cache_len int32 [B] (device) the sequences' lengths (query at cache_len - 1)."""
    import torch
    B, H, d = q.shape
    cap = kcache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = load().pi_attn_decode_ring(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(w_g), _ptr(b_g), _ptr(cache_len),
                                    _ptr(out), _ptr(lse), B, H, cap, d, k_win, pi, S, _dtype_code(q), _stream(stream))
    _raise(st)
    return out, lse


def pi_attn_cache_append(kcache, vcache, k_new, v_new, cache_len, *, ring: bool = True, stream=None):
    """Append one token per (b, h) (k_new, v_new [B, H, d]) at position cache_len[b], then advance
    cache_len.  The caches are [B, H, capacity, d]; ring: slot = position mod capacity."""
    B, H, cap, d = kcache.shape
    st = load().pi_attn_cache_append(_ptr(kcache), _ptr(vcache), _ptr(k_new), _ptr(v_new), _ptr(cache_len), B, H, cap,
                                     d, _dtype_code(kcache), int(ring), _stream(stream))
    _raise(st)


def pi_attn_check(stream=None):
    """Synchronise the stream and raise if a kernel set the device error word."""
    _raise(load().pi_attn_check(_stream(stream)))


def pi_attn_version() -> int:
    return load().pi_attn_version()
