"""Out-of-bounds writes (B200 only): every output a call writes sits inside a larger device buffer
whose guard regions before and after it hold a fixed bit pattern; after the call the guards must
be unchanged.  The shapes are ragged (rows not a multiple of the 128-row tile, sequences not a
whole number of periods), so tile stores clipped by the tensor maps, the split path's tail, the
split decode's partials and the host-buffer entry points' chunk buffers (inside the caller's
workspace) are all exercised at their edges.
"""
import math

import numpy as np
import pytest
import torch

import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

GUARD_BYTES = 8192
PATTERN = {torch.bfloat16: -16447, torch.float32: 0x7FC12345, torch.uint8: 0xA5}  # NaN bits / a byte pattern


@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()
    pia.load()
    yield
    torch.cuda.synchronize()


class Guarded:
    """A device tensor of `shape` inside a buffer with GUARD_BYTES of pattern on each side."""

    def __init__(self, shape, dtype):
        self.dtype = dtype
        esize = torch.tensor([], dtype=dtype).element_size()
        self.g = GUARD_BYTES // esize
        numel = int(np.prod(shape))
        self.buf = torch.empty(numel + 2 * self.g, dtype=dtype, device="cuda")
        self._bits().fill_(PATTERN[dtype])
        self.t = self.buf[self.g:self.g + numel].view(shape)

    def _bits(self):
        if self.dtype == torch.bfloat16:
            return self.buf.view(torch.int16)
        if self.dtype == torch.float32:
            return self.buf.view(torch.int32)
        return self.buf

    def check(self, what):
        torch.cuda.synchronize()
        bits = self._bits()
        for name, part in (("before", bits[:self.g]), ("after", bits[-self.g:])):
            bad = int((part != PATTERN[self.dtype]).sum())
            assert bad == 0, f"{what}: {bad} guard elements {name} the output were written"


def _inputs(B, H, n, d, dtype, seed):
    dev = {x: to_dev(ps.normal((B, H, n, d), seed=seed, stream=s, dtype=dtype), dtype)
           for x, s in (("q", 1), ("k", 2), ("v", 3), ("dO", 6))}
    dev["w_g"] = torch.from_numpy(ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32")).cuda()
    dev["b_g"] = torch.from_numpy(ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")).cuda()
    return dev


FWD_CASES = [  # B, H, n, d, k, pi, S, dtype, path
    (2, 3, 1000, 64, 40, 16, 30, "bf16", "tc_fused"),     # ragged rows, many skips
    (1, 2, 2100, 128, 100, 128, 12, "bf16", "auto"),      # the split path with a tail past the periods
    (2, 2, 300, 32, 20, 9, 5, "f32", "auto"),             # the CUDA-core kernel
]


@pytest.mark.parametrize("case", FWD_CASES, ids=[f"{c[7]}-{c[8]}-n{c[2]}" for c in FWD_CASES])
def test_prefill_writes_only_its_outputs(case):
    B, H, n, d, k, pi, S, dtype, path = case
    x = _inputs(B, H, n, d, dtype, seed=n)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out, lse = Guarded((B, H, n, d), tdt), Guarded((B, H, n), torch.float32)
    pia.pi_attn_fwd(x["q"], x["k"], x["v"], x["w_g"], x["b_g"], k, pi, S, out=out.t, lse=lse.t, path=path)
    pia.pi_attn_check()
    out.check(f"{case} out")
    lse.check(f"{case} lse")
    assert bool(torch.isfinite(out.t.float()).all()) and bool(torch.isfinite(lse.t).all())


def test_split_decode_writes_only_its_outputs():
    # few (b, h): the decode splits each cache across CTAs and combines their partials
    B, H, n_cache, d, k, pi, S = 1, 4, 9000, 128, 1024, 2048, 31
    q = to_dev(ps.normal((B, H, d), seed=1, stream=11, dtype="bf16"), "bf16")
    kc = to_dev(ps.normal((B, H, n_cache, d), seed=1, stream=12, dtype="bf16"), "bf16")
    vc = to_dev(ps.normal((B, H, n_cache, d), seed=1, stream=13, dtype="bf16"), "bf16")
    wg = torch.from_numpy(ps.normal((H, d), seed=1, stream=14, std=1 / math.sqrt(d), dtype="f32")).cuda()
    bg = torch.zeros(H, device="cuda")
    out, lse = Guarded((B, H, d), torch.bfloat16), Guarded((B, H), torch.float32)
    pia.pi_attn_decode(q, kc, vc, wg, bg, k, pi, S, out=out.t, lse=lse.t)
    pia.pi_attn_check()
    out.check("decode out")
    lse.check("decode lse")


@pytest.mark.parametrize("path", ["tc_fused", "tc_split", "simt"])
def test_backward_writes_only_its_gradients(path):
    B, H, n, d, k, pi, S = 2, 2, 2560, 64, 50, 10, 20  # n a whole number of periods (the split needs it)
    x = _inputs(B, H, n, d, "bf16", seed=4)
    grads = [Guarded((B, H, n, d), torch.float32) for _ in range(3)] + \
        [Guarded((H, d), torch.float32), Guarded((H,), torch.float32)]
    pia.pi_attn_bwd(x["q"], x["k"], x["v"], x["w_g"], x["b_g"], x["dO"], k, pi, S, grads=tuple(g.t for g in grads),
                    path=path)
    pia.pi_attn_check()
    for name, g in zip(("dq", "dk", "dv", "dw_g", "db_g"), grads):
        g.check(f"{path} {name}")


def test_host_entry_points_stay_inside_their_workspace():
    # the chunk buffers of the host-buffer entry points live in the caller's workspace: the guard
    # after the workspace's last byte must survive a ragged last chunk
    B, H, n, d, k, pi, S = 1, 5, 1100, 64, 40, 100, 5
    x = _inputs(B, H, n, d, "bf16", seed=9)
    host = {name: x[name].cpu().pin_memory() for name in ("q", "k", "v", "dO")}
    nb = pia.pi_attn_fwd_host_workspace_bytes(B, H, n, d, "bf16", 2)
    ws = Guarded((nb,), torch.uint8)
    pia.pi_attn_fwd_host(host["q"], host["k"], host["v"], x["w_g"], x["b_g"], k, pi, S, chunk_heads=2,
                         workspace=ws.t)
    pia.pi_attn_check()
    ws.check("pi_attn_fwd_host workspace")
    nb = pia.load().pi_attn_bwd_host_workspace_bytes(B, H, n, d, pia.PI_ATTN_BF16, pia.BWD_PATHS["tc"], 2)
    ws = Guarded((nb,), torch.uint8)
    gw, gb = Guarded((H, d), torch.float32), Guarded((H,), torch.float32)
    grads = tuple(torch.empty((B, H, n, d), dtype=torch.float32).pin_memory() for _ in range(3)) + (gw.t, gb.t)
    pia.pi_attn_bwd_host(host["q"], host["k"], host["v"], x["w_g"], x["b_g"], host["dO"], k, pi, S, grads=grads,
                         path="tc", chunk_heads=2, workspace=ws.t)
    pia.pi_attn_check()
    ws.check("pi_attn_bwd_host workspace")
    gw.check("pi_attn_bwd_host dw_g")
    gb.check("pi_attn_bwd_host db_g")
