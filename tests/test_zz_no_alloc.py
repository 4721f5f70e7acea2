"""pi_attn_decode_noalloc: decode for callers that cannot allocate device memory (B200 only).

Some callers cannot let a library allocate. A process that reserves its device memory up front
with its own allocator has no headroom for a library allocation. A runtime with a fixed memory
plan must account for every byte in advance. For them the library offers a decode entry point
whose workspace is a fixed array inside the library instead of cudaMallocAsync memory.

This test calls that entry point through the C ABI. It compares the results with
pi_attn_decode's on the same inputs, within the parity tolerances of the bf16 tests. It does so
for two calls in a row with different problems, so a stale workspace from the first call would
show in the second. The shapes are chosen so that the work is split across CTAs: that is the
case that uses the workspace.
This file sorts last, so a run that stops at the first failure has run every other test first.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from tests.gpu_util import TOL, assert_close, from_dev, metrics, to_dev

pytestmark = pytest.mark.gpu


def _problem(B, H, n_cache, d, seed):
    q = to_dev(ps.normal((B, H, d), seed=seed, stream=11), "bf16")
    kc = to_dev(ps.normal((B, H, n_cache, d), seed=seed, stream=12), "bf16")
    vc = to_dev(ps.normal((B, H, n_cache, d), seed=seed, stream=13), "bf16")
    w_g = torch.from_numpy(ps.normal((H, d), seed=seed, stream=14, std=1 / math.sqrt(d), dtype="f32")).cuda()
    b_g = torch.from_numpy(ps.normal((H,), seed=seed, stream=15, std=0.7, dtype="f32")).cuda()
    return q, kc, vc, w_g, b_g


def _call(fn, q, kc, vc, w_g, b_g, cache_len, k, pi, S):
    B, H, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = fn(p(q), p(kc), p(vc), p(w_g), p(b_g), p(cache_len), p(out), p(lse), B, H, kc.shape[2], d, k, pi, S,
            pia.PI_ATTN_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pia.PI_ATTN_OK, pia.load().pi_attn_last_error()
    return out, lse


# (B, H, n_cache, d, k_win, pi, S, cache lengths or None): few (b, h), so the work is split
CASES = [
    (1, 4, 9000, 128, 1024, 2048, 31, None),
    (2, 3, 20000, 64, 3000, 700, 25, [20000, 7777]),
]


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row():
    pbuild.build()
    lib = pia.load()
    for seed, (B, H, n_cache, d, k, pi, S, lengths) in enumerate(CASES):
        q, kc, vc, w_g, b_g = _problem(B, H, n_cache, d, seed=100 + seed)
        cl = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device="cuda")
        ref_out, ref_lse = _call(lib.pi_attn_decode, q, kc, vc, w_g, b_g, cl, k, pi, S)
        out, lse = _call(lib.pi_attn_decode_noalloc, q, kc, vc, w_g, b_g, cl, k, pi, S)
        pia.pi_attn_check()
        m = metrics(from_dev(out).reshape(B * H, d), from_dev(ref_out).reshape(B * H, d),
                    lse.cpu().numpy().astype(np.float64).reshape(-1), ref_lse.cpu().numpy().astype(np.float64).reshape(-1))
        assert_close(m, "bf16", f"no-alloc decode, call {seed + 1}")
    assert TOL["bf16"]["out_abs"] == 2e-2  # the parity tolerance of the bf16 tests
