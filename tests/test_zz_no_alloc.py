"""pi_attn_decode_noalloc: decode for callers that cannot allocate device memory (B200 only).

Some callers cannot let a library allocate. A process that reserves its device memory up front
with its own allocator has no headroom for a library allocation. A runtime with a fixed memory
plan must account for every byte in advance. For them the library offers a decode entry point
whose workspace is a fixed array inside the library instead of cudaMallocAsync memory.

This test calls that entry point through the C ABI, for two calls in a row with different
problems, so a stale workspace from the first call would show in the second. The shapes are
chosen so that the work is split across CTAs: that is the case that uses the workspace.

- It runs the same kernels as pi_attn_decode on the same inputs, so its results must be the
  same bits.
- Both are compared with the fp64 decode oracle, within the parity tolerances of the bf16 tests.
- It must allocate nothing: the high watermark of the device's current memory pool (where
  cudaMallocAsync takes its memory) is reset before each call and read after it. pi_attn_decode
  raises it on these shapes; pi_attn_decode_noalloc must leave it where it was.

This file sorts last, so a run that stops at the first failure has run every other test first.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from tests.gpu_util import assert_close, from_dev, metrics, to_dev

pytestmark = pytest.mark.gpu


def _problem(B, H, n_cache, d, seed):
    host = {"q": ps.normal((B, H, d), seed=seed, stream=11),
            "kc": ps.normal((B, H, n_cache, d), seed=seed, stream=12),
            "vc": ps.normal((B, H, n_cache, d), seed=seed, stream=13),
            "w_g": ps.normal((H, d), seed=seed, stream=14, std=1 / math.sqrt(d), dtype="f32"),
            "b_g": ps.normal((H,), seed=seed, stream=15, std=0.7, dtype="f32")}
    dev = {x: to_dev(host[x], "bf16") for x in ("q", "kc", "vc")}
    dev["w_g"] = torch.from_numpy(host["w_g"]).cuda()
    dev["b_g"] = torch.from_numpy(host["b_g"]).cuda()
    return host, dev


class _PoolWatermark:
    """The high watermark of the memory pool cudaMallocAsync draws from on the current device
    (driver API through cuda-python; it only reads and resets the pool's usage statistic)."""

    def __init__(self):
        from cuda.bindings import driver as cu
        self.cu = cu
        (err,) = cu.cuInit(0)
        assert err == cu.CUresult.CUDA_SUCCESS, err
        err, self.pool = cu.cuDeviceGetMemPool(torch.cuda.current_device())
        assert err == cu.CUresult.CUDA_SUCCESS, err
        self.attr = cu.CUmemPool_attribute.CU_MEMPOOL_ATTR_USED_MEM_HIGH

    def reset(self):
        (err,) = self.cu.cuMemPoolSetAttribute(self.pool, self.attr, self.cu.cuuint64_t(0))
        assert err == self.cu.CUresult.CUDA_SUCCESS, err

    def high(self) -> int:
        err, v = self.cu.cuMemPoolGetAttribute(self.pool, self.attr)
        assert err == self.cu.CUresult.CUDA_SUCCESS, err
        return int(v)


def _call(fn, dev, cache_len, k, pi, S, out, lse):
    B, H, d = dev["q"].shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = fn(p(dev["q"]), p(dev["kc"]), p(dev["vc"]), p(dev["w_g"]), p(dev["b_g"]), p(cache_len), p(out), p(lse), B, H,
            dev["kc"].shape[2], d, k, pi, S, pia.PI_ATTN_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pia.PI_ATTN_OK, pia.load().pi_attn_last_error()


# (B, H, n_cache, d, k_win, pi, S, cache lengths or None): few (b, h), so the work is split
CASES = [
    (1, 4, 9000, 128, 1024, 2048, 31, None),
    (2, 3, 20000, 64, 3000, 700, 25, [20000, 7777]),
]


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row():
    pbuild.build()
    lib = pia.load()
    pool = _PoolWatermark()
    for seed, (B, H, n_cache, d, k, pi, S, lengths) in enumerate(CASES):
        host, dev = _problem(B, H, n_cache, d, seed=100 + seed)
        cl = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device="cuda")
        ref_out, out = torch.empty_like(dev["q"]), torch.empty_like(dev["q"])
        ref_lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        lse = torch.empty_like(ref_lse)
        torch.cuda.synchronize()

        pool.reset()
        _call(lib.pi_attn_decode, dev, cl, k, pi, S, ref_out, ref_lse)
        torch.cuda.synchronize()
        assert pool.high() > 0, "pi_attn_decode took no workspace: the shape does not split"

        pool.reset()
        base = pool.high()
        _call(lib.pi_attn_decode_noalloc, dev, cl, k, pi, S, out, lse)
        torch.cuda.synchronize()
        assert pool.high() == base, f"pi_attn_decode_noalloc allocated (pool high {base} -> {pool.high()})"
        pia.pi_attn_check()

        # the same kernels on the same inputs: the same bits
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"call {seed + 1}: out differs"
        assert torch.equal(lse, ref_lse), f"call {seed + 1}: lse differs"

        # and both within the bf16 parity tolerances of the fp64 oracle
        ro, rl, _ = oracle.decode(host["q"], host["kc"], host["vc"], host["w_g"], host["b_g"], k, pi, S,
                                  lengths=None if lengths is None else np.asarray(lengths, np.int32))
        m = metrics(from_dev(out).reshape(B * H, d), ro, lse.cpu().numpy().astype(np.float64).reshape(-1), rl)
        assert_close(m, "bf16", f"no-alloc decode against the oracle, call {seed + 1}")
