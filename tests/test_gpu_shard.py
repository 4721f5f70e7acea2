"""Sequence sharding on the GPU (B200 only): pi_attn_fwd_shard over each rank's rows, the halo
taken from the whole sequence the way the exchange delivers it, against the fp64 oracle on the
whole sequence.  The ranks run one after another on one device (no kernel waits on another); the
exchange itself is tested between gloo ranks in test_shard.py."""
import math

import numpy as np
import pytest
import torch

import oracle
import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from periodic_sparse_attention_b200 import shard
from tests.gpu_util import assert_close, from_dev, metrics, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()
    pia.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()


def _inputs(B, H, n, d, seed):
    q = ps.normal((B, H, n, d), seed=seed, stream=1, dtype="bf16")
    k = ps.normal((B, H, n, d), seed=seed, stream=2, dtype="bf16")
    v = ps.normal((B, H, n, d), seed=seed, stream=3, dtype="bf16")
    w_g = ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")
    return q, k, v, w_g, b_g


def _run_shards(qt, kt, vt, wg, bg, n, world, kw, pi, S, halo_from_zero=False, align=1):
    outs, lses = [], []
    for r in range(world):
        s0, s1 = shard.shard_bounds(n, world, r, align)
        if s1 == s0:
            continue
        kv0 = 0 if halo_from_zero else shard.halo_start(s0, s1, kw, pi, S, align)
        o, l = pia.pi_attn_fwd_shard(qt[:, :, s0:s1].contiguous(), kt[:, :, kv0:s1].contiguous(),
                                     vt[:, :, kv0:s1].contiguous(), wg, bg, kw, pi, S, s0, kv0)
        outs.append(o)
        lses.append(l)
    pia.pi_attn_check()
    return torch.cat(outs, dim=2), torch.cat(lses, dim=2)


@pytest.mark.parametrize("case", [
    # B, H, n, d, k, pi, S, world
    (1, 2, 1000, 64, 40, 16, 30, 4),      # halo of 480 rows: reaches two ranks back
    (2, 2, 777, 128, 100, 7, 40, 3),      # ragged shards, rows not 128-aligned
    (1, 3, 4096, 64, 128, 64, 4, 4),      # the bf16_n4k geometry in four shards
    (1, 1, 2500, 128, 256, 256, 8, 2),    # the bf16_n32k geometry, shorter
    (1, 2, 300, 64, 8, 16, 2, 5),         # short shards (60 rows)
    # shards of whole periods with halos of whole periods: every rank takes the split path (the
    # residue pass and the window pass with the shard's offsets)
    (1, 2, 8192, 64, 128, 256, 16, 4),    # halos of 4096 rows, reaching two ranks back
    (2, 2, 6144, 128, 256, 512, 8, 3),    # d = 128, halo to row 0
])
def test_shards_match_the_oracle_on_the_whole_sequence(case):
    B, H, n, d, kw, pi, S, world = case
    q, k, v, w_g, b_g = _inputs(B, H, n, d, seed=n + world)
    qt, kt, vt = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    wg, bg = torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda()
    out, lse = _run_shards(qt, kt, vt, wg, bg, n, world, kw, pi, S)
    ro, rl = oracle.fwd(q, k, v, w_g, b_g, kw, pi, S)[:2]
    assert_close(metrics(from_dev(out).reshape(-1, d), ro.reshape(-1, d), lse.cpu().numpy().astype(np.float64).reshape(-1),
                         rl.reshape(-1)), "bf16", str(case))
    # a halo reaching back to row 0 holds more rows than the shard reads; the result is the same
    # up to rounding (a tile's reference maximum also sees the masked keys, which the shorter
    # halo zero-fills before its first row)
    out0, lse0 = _run_shards(qt, kt, vt, wg, bg, n, world, kw, pi, S, halo_from_zero=True)
    assert_close(metrics(from_dev(out0).reshape(-1, d), ro.reshape(-1, d),
                         lse0.cpu().numpy().astype(np.float64).reshape(-1), rl.reshape(-1)), "bf16", f"{case} full halo")


@pytest.mark.parametrize("d", [64, 128])
def test_one_shard_is_the_single_pass_forward(d):
    B, H, n, kw, pi, S = 1, 2, 1500, 100, 32, 9
    q, k, v, w_g, b_g = _inputs(B, H, n, d, seed=3)
    qt, kt, vt = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    wg, bg = torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda()
    o1, l1 = pia.pi_attn_fwd_shard(qt, kt, vt, wg, bg, kw, pi, S, 0, 0)
    o2, l2 = pia.pi_attn_fwd(qt, kt, vt, wg, bg, kw, pi, S, path="tc_fused")
    pia.pi_attn_check()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
def test_a_whole_sequence_shard_takes_the_split_path(d):
    # a shard that is the whole sequence, on a shape that takes the split path, runs the same
    # launches as the whole-sequence forward: the same bits
    B, H, n, kw, pi, S = 1, 2, 4096, 128, 256, 12
    assert pia.pi_attn_fwd_plan(B, H, n, d, kw, pi, S, "bf16", "auto")[0] >= 2  # the split path
    q, k, v, w_g, b_g = _inputs(B, H, n, d, seed=11)
    qt, kt, vt = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    wg, bg = torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda()
    o1, l1 = pia.pi_attn_fwd_shard(qt, kt, vt, wg, bg, kw, pi, S, 0, 0)
    o2, l2 = pia.pi_attn_fwd(qt, kt, vt, wg, bg, kw, pi, S)
    pia.pi_attn_check()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_shards_on_whole_periods_take_the_split_path_and_match_the_oracle():
    # three ranks on a sequence that is not a whole number of periods: blocks and halos aligned to
    # whole periods (the layout bench.py --shard seq uses), so every rank takes the split path and
    # the last rank's tail its single pass
    B, H, n, d, kw, pi, S, world = 1, 2, 20 * 1024 + 300, 128, 512, 1024, 12, 3  # the last halo from row 2048
    q, k, v, w_g, b_g = _inputs(B, H, n, d, seed=17)
    qt, kt, vt = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    wg, bg = torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda()
    out, lse = _run_shards(qt, kt, vt, wg, bg, n, world, kw, pi, S, align=pi)
    ro, rl = oracle.fwd(q, k, v, w_g, b_g, kw, pi, S)[:2]
    assert_close(metrics(from_dev(out).reshape(-1, d), ro.reshape(-1, d), lse.cpu().numpy().astype(np.float64).reshape(-1),
                         rl.reshape(-1)), "bf16", "aligned shards")


def test_shard_with_a_workspace_gives_the_same_bits():
    # pi_attn_fwd_shard_ws with the caller's workspace and pi_attn_fwd_shard with its own scratch:
    # the same launches, the same bits (a shard of whole periods with a halo: the split path)
    import ctypes
    B, H, n, d, kw, pi, S = 1, 2, 8192, 64, 128, 256, 16
    q, k, v, w_g, b_g = _inputs(B, H, n, d, seed=23)
    qt, kt, vt = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    wg, bg = torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda()
    s0, s1, kv0 = 4096, 8192, 0
    need = pia.load().pi_attn_fwd_shard_scratch_bytes(B, H, s1 - s0, s0, kv0, d, kw, pi, S)
    assert need > 0
    qs, ks, vs = qt[:, :, s0:s1].contiguous(), kt[:, :, kv0:s1].contiguous(), vt[:, :, kv0:s1].contiguous()
    o1, l1 = pia.pi_attn_fwd_shard(qs, ks, vs, wg, bg, kw, pi, S, s0, kv0)  # the binding's workspace
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = pia.load().pi_attn_fwd_shard(P(qs), P(ks), P(vs), P(wg), P(bg), P(o2), P(l2), B, H, s1 - s0, s1 - kv0, s0,
                                      kv0, d, kw, pi, S, pia.PI_ATTN_BF16,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))  # its own scratch
    assert st == pia.PI_ATTN_OK, pia.load().pi_attn_last_error()
    pia.pi_attn_check()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)
