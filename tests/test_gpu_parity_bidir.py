"""Bidirectional variant on the GPU against the fp64 oracle, through the C ABI (B200 only).

The rule: the window reaches k tokens both ways, [max(0, i - k), min(n - 1, i + k)], and every
surviving m adds a forward skip i + m*pi next to the backward one (pi_attn_fwd_bidir).  Small
cases compare every row; the long case compares sampled rows plus the rows at both ends of every
(b, h), where the two directions are cut by the sequence bounds.
"""
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


@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()
    pia.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()


def _inputs(B, H, n, d, dtype, seed):
    return {"q": ps.normal((B, H, n, d), seed=seed, stream=1, dtype=dtype),
            "k": ps.normal((B, H, n, d), seed=seed, stream=2, dtype=dtype),
            "v": ps.normal((B, H, n, d), seed=seed, stream=3, dtype=dtype),
            "w_g": ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32"),
            "b_g": ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")}


def _run(inp, dtype, k, pi, S, path):
    q, kk, v = (to_dev(inp[x], dtype) for x in ("q", "k", "v"))
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    out, lse = pia.pi_attn_fwd(q, kk, v, wg, bg, k, pi, S, path=path, bidir=True)
    pia.pi_attn_check()
    return from_dev(out), lse.cpu().numpy().astype(np.float64)


CASES = [  # B, H, n, d, k, pi, S
    (1, 1, 1, 64, 0, 1, 1),          # a single token
    (2, 3, 1000, 128, 100, 37, 12),  # ragged tail, many skips both ways
    (1, 2, 333, 64, 400, 16, 40),    # window longer than the sequence (every key, once)
    (1, 1, 200, 128, 64, 32, 0),     # no skips: two-sided sliding window
    (1, 1, 300, 64, 8, 1, 50),       # period 1
    (1, 2, 513, 128, 128, 64, 6),    # ties m*pi == k
    (1, 1, 130, 64, 5, 7, 3),        # tiny window, ragged
    (2, 2, 640, 128, 0, 128, 4),     # window of the token alone
    (1, 1, 4096, 64, 128, 64, 4),    # the bf16_n4k shape
    (1, 1, 2112, 64, 10, 64, 40),    # forward skips reach the end from most rows
]


def _bidir_split_applies(n, k, pi, S, d):
    # the bidirectional split: n a whole number of periods, a skip outside the window
    return d in (64, 128) and n % pi == 0 and S >= k // pi + 1


@pytest.mark.parametrize("path", ["auto", "simt", "tc_fused", "tc_split"])
@pytest.mark.parametrize("case", CASES)
def test_bidir_bf16_every_row(case, path):
    B, H, n, d, k, pi, S = case
    if path == "tc_split" and not _bidir_split_applies(n, k, pi, S, d):
        pytest.skip("the bidirectional split needs n % pi == 0 and a skip outside the window")
    inp = _inputs(B, H, n, d, "bf16", seed=3 * n + k)
    out, lse = _run(inp, "bf16", k, pi, S, path)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S, bidir=True)
    assert_close(metrics(out, ro, lse, rl), "bf16", f"bidir {case}/{path}")


@pytest.mark.parametrize("case", [(1, 1, 1, 32, 0, 1, 1), (2, 3, 257, 32, 8, 16, 2), (1, 2, 300, 128, 40, 9, 7),
                                  (1, 1, 100, 4, 3, 2, 5)])
def test_bidir_f32_every_row(case):
    B, H, n, d, k, pi, S = case
    inp = _inputs(B, H, n, d, "f32", seed=n + 5 * k)
    out, lse = _run(inp, "f32", k, pi, S, "auto")
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S, bidir=True)
    assert_close(metrics(out, ro, lse, rl), "f32", f"bidir {case}")


@pytest.mark.parametrize("path", ["auto", "tc_fused", "tc_split"])
def test_bidir_long_sequence_sampled_rows(path):
    # the bf16_n32k shape under the bidirectional rule; auto takes the split (both skip bands in the
    # residue-class pass, the two-sided window in the band-merge pass)
    B, H, n, d, k, pi, S = 2, 16, 32768, 128, 256, 256, 8
    assert pia.pi_attn_fwd_plan(B, H, n, d, k, pi, S, "bf16", "auto")[0] == 2  # the causal rule splits this shape too
    inp = _inputs(B, H, n, d, "bf16", seed=41)
    out, lse = _run(inp, "bf16", k, pi, S, path)
    rng = np.random.default_rng(0)
    rows = rng.choice(B * H * n, 2048, replace=False)
    ends = [bh * n + i for bh in range(B * H) for i in (0, k, pi, n - 1 - pi, n - 1 - k, n - 1)]
    rows = np.unique(np.concatenate([rows, np.array(ends)]))
    ro, rl, _ = oracle.fwd_rows(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S, rows=rows, bidir=True)
    assert_close(metrics(out.reshape(-1, d)[rows], ro, lse.reshape(-1)[rows], rl), "bf16", f"bidir n32k/{path}")
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def test_bidir_reversal_symmetry_on_the_gpu():
    # reversing the sequence reverses the result (up to rounding): both directions are symmetric
    B, H, n, d, k, pi, S = 1, 4, 1500, 64, 70, 48, 9
    inp = _inputs(B, H, n, d, "bf16", seed=43)
    out, lse = _run(inp, "bf16", k, pi, S, "auto")
    rev = {x: np.ascontiguousarray(inp[x][:, :, ::-1]) for x in ("q", "k", "v")}
    rev.update(w_g=inp["w_g"], b_g=inp["b_g"])
    out_r, lse_r = _run(rev, "bf16", k, pi, S, "auto")
    assert np.max(np.abs(out_r[:, :, ::-1] - out)) <= 2e-2
    assert np.max(np.abs(lse_r[:, :, ::-1] - lse)) <= 1e-3


@pytest.mark.parametrize("n,k,pi,S", [(1000, 8, 16, 2), (4096, 128, 64, 4), (777, 0, 1, 70), (500, 600, 7, 3),
                                      (300, 20, 5, 0), (2000, 100, 300, 9)])
def test_bidir_index_sets_bit_exact(n, k, pi, S):
    c, idx = pia.pi_attn_debug_index_sets(n, k, pi, S, bidir=True)
    torch.cuda.synchronize()
    rc, ridx = oracle.index_table(n, k, pi, S, bidir=True)
    assert np.array_equal(c.cpu().numpy(), rc)
    assert np.array_equal(idx.cpu().numpy(), ridx)


def test_bidir_split_path_needs_whole_periods():
    # a forward skip may reach past the last whole period, outside the residue view: refused before
    # any launch; on a whole number of periods the split runs and matches the oracle
    inp = _inputs(1, 1, 250, 64, "bf16", seed=1)
    q, kk, v = (to_dev(inp[x], "bf16") for x in ("q", "k", "v"))
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    with pytest.raises(pia.PiAttnError) as e:
        pia.pi_attn_fwd(q, kk, v, wg, bg, 8, 64, 3, path="tc_split", bidir=True)
    assert e.value.status == pia.PI_ATTN_EUNSUPPORTED
    pia.pi_attn_check()  # nothing was launched: the stream is still clean
    inp = _inputs(1, 2, 256, 64, "bf16", seed=1)
    out, lse = _run(inp, "bf16", 8, 64, 3, "tc_split")
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], 8, 64, 3, bidir=True)
    assert_close(metrics(out, ro, lse, rl), "bf16", "bidir split n256")
