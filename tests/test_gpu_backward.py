"""The backward (pi_attn_bwd, and pi_attn_bwd_ex with the tensor-core dq pass) on the GPU against
the fp64 backward oracle (B200 only).

Every element of dq, dk, dv, dw_g and db_g is compared.  Inputs are identical bits on both sides,
so the differences are the GPU's fp32 accumulation against the oracle's fp64; the bound, written
in tests/gpu_util.py (grad_close), is a relative L2 error and a max-abs error as a fraction of the
gradient's largest magnitude, for every gradient.  The gate gradients dw_g and db_g are sums over
every row of dz_i, a sum of terms that cancel (to exactly zero on a row whose keys all carry the
same prior); they are held to a rounding bound formed from the oracle's per-row terms
(tests/gpu_util.py gate_scales), which also covers problems whose true gate gradients are zero.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from tests.gpu_util import gate_scales, grad_close, to_dev

pytestmark = pytest.mark.gpu

# Bounds per path (fp32 CUDA-core path; tensor-core path): tests/gpu_util.py GRAD_TOL.

@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()
    pia.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()


def _problem(B, H, n, d, dtype, seed):
    return {"q": ps.normal((B, H, n, d), seed=seed, stream=1, dtype=dtype),
            "k": ps.normal((B, H, n, d), seed=seed, stream=2, dtype=dtype),
            "v": ps.normal((B, H, n, d), seed=seed, stream=3, dtype=dtype),
            "w_g": ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32"),
            "b_g": ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32"),
            "dO": ps.normal((B, H, n, d), seed=seed, stream=6, dtype=dtype)}


def _widen(a):
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if a.dtype == np.uint16 else \
        a.astype(np.float64)


def _check(inp, dtype, k, pi, S, bidir, what, path="simt"):
    dev = {x: to_dev(inp[x], dtype) for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    got = pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], k, pi, S, bidir=bidir, path=path)
    pia.pi_attn_check()
    *ref, terms = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], _widen(inp["dO"]), k, pi, S,
                             bidir=bidir, return_terms=True)
    rss_dw, rss_db = gate_scales(inp["q"], terms)
    for name, g, r in zip(["dq", "dk", "dv", "dw_g", "db_g"], got, ref):
        g = g.cpu().numpy().astype(np.float64)
        ok, msg = grad_close(name, g, r, "simt" if path == "simt" else "tc",
                             rss_dw if name == "dw_g" else rss_db if name == "db_g" else None)
        assert ok, f"{what}: {msg}"
    return got, ref


CASES = [  # B, H, n, d, k, pi, S
    (1, 2, 64, 32, 8, 16, 2),
    (2, 3, 300, 64, 20, 9, 5),      # ragged, many skips
    (1, 2, 513, 128, 128, 64, 6),   # ties m*pi == k
    (1, 1, 1, 64, 0, 1, 1),         # a single token
    (1, 2, 200, 64, 300, 16, 20),   # window longer than the sequence
    (1, 1, 150, 32, 5, 1, 30),      # period 1
    (1, 2, 128, 64, 16, 32, 0),     # no skips
]


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", CASES)
def test_backward_every_element(case, dtype, bidir):
    B, H, n, d, k, pi, S = case
    _check(_problem(B, H, n, d, dtype, seed=n + 13 * k), dtype, k, pi, S, bidir, f"{case} {dtype} bidir={bidir}")


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("case", [c for c in CASES if c[3] in (64, 128)] + [(1, 2, 1000, 128, 100, 37, 12)])
def test_backward_tensor_core_path(case, bidir):
    B, H, n, d, k, pi, S = case
    _check(_problem(B, H, n, d, "bf16", seed=n + 13 * k), "bf16", k, pi, S, bidir, f"{case} tc bidir={bidir}",
           path="tc")


# The split backward: causal, n a whole number of periods, skips outside the window.  The residue
# view has T = n / pi rows per class: fewer than a 128-row tile, one tile, several with a ragged
# last one; pi = 1 (the view is the sequence); a skip band wider than a key tile.
SPLIT_CASES = [  # B, H, n, d, k, pi, S
    (1, 1, 64, 64, 8, 16, 3),          # T = 4
    (1, 2, 1024, 64, 40, 16, 30),      # T = 64, 28 skips
    (2, 2, 2048, 128, 100, 64, 12),    # T = 32, m0 = 2
    (1, 1, 8192, 128, 256, 32, 40),    # T = 256: two row tiles per class, m0 = 9
    (1, 2, 3000, 64, 10, 1, 90),       # pi = 1: the band of 80 skips is the sequence's
    (1, 2, 2560, 64, 50, 10, 20),      # T = 256, m0 = 6
    (1, 1, 4480, 128, 200, 35, 7),     # T = 128, m0 = 6: two skips
    (1, 1, 2048, 64, 64, 32, 6),       # tie: 2 * pi == k is a window key, m0 = 3
]


@pytest.mark.parametrize("case", SPLIT_CASES)
@pytest.mark.parametrize("path", ["tc_split", "tc_fused"])
def test_backward_tensor_core_split_and_fused(case, path):
    B, H, n, d, k, pi, S = case
    _check(_problem(B, H, n, d, "bf16", seed=n + 7 * S), "bf16", k, pi, S, False, f"{case} {path}", path=path)


def test_backward_split_n4k_geometry_and_determinism():
    # the bf16_n4k shape (pi = 64, T = 64) through the split passes, twice: the same bits
    w = ps.WORKLOADS["bf16_n4k"]
    inp = ps.prefill_inputs(w)
    inp["dO"] = ps.normal((w.B, w.H, w.n, w.d), seed=0, stream=6, dtype="bf16")
    a = [t.clone() for t in _check(inp, "bf16", w.k, w.pi, w.S, False, "bf16_n4k tc_split", path="tc_split")[0]]
    dev = {x: to_dev(inp[x], "bf16") for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    b = pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], w.k, w.pi, w.S, path="tc_split")
    pia.pi_attn_check()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_split_bf16_n32k_workload_one_sequence():
    # one (b, h) sequence of the bf16_n32k_bwd workload at its full length, through the split path
    # the bench's tc path takes there, every element against the oracle
    w = ps.WORKLOADS["bf16_n32k_bwd"]
    inp = ps.backward_inputs(w)
    one = {x: np.ascontiguousarray(inp[x][:1, :1]) for x in ("q", "k", "v", "dO")}
    one["w_g"], one["b_g"] = inp["w_g"][:1], inp["b_g"][:1]
    _check(one, "bf16", w.k, w.pi, w.S, False, "bf16_n32k_bwd (0, 0) tc_split", path="tc_split")


@pytest.mark.parametrize("workload", ["bf16_n32k_bwd", "bf16_n4k_bwd"])
def test_backward_full_workload_gradient_sums(workload):
    # The whole workload in the bench's launch configuration (path tc: the split passes on
    # bf16_n32k_bwd), every (b, h) and column, against two closed forms of the method: a row's
    # weights sum to one, so sum_j dv_j = sum_i dO_i, and a row's ds sum to zero, so sum_j dk_j = 0.
    # The bounds allow the bf16 roundings of P and ds (relative 2^-9 each, summed with random
    # signs): 4e-3 of the column norm of dO, and 1e-2 of the column norm of dk.
    w = ps.WORKLOADS[workload]
    inp = ps.backward_inputs(w)
    dev = {x: to_dev(inp[x], "bf16") for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    _, dk, dv, dw, db = pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], w.k, w.pi, w.S, path="tc")
    pia.pi_attn_check()
    assert bool(torch.isfinite(dw).all()) and bool(torch.isfinite(db).all())
    dO = dev["dO"].double()
    ev = (dv.double().sum(dim=2) - dO.sum(dim=2)).abs() / dO.norm(dim=2)
    assert float(ev.max()) <= 4e-3, float(ev.max())
    dk = dk.double()
    ek = dk.sum(dim=2).abs() / dk.norm(dim=2).clamp_min(1e-30)
    assert float(ek.max()) <= 1e-2, float(ek.max())


def test_backward_tensor_core_path_bf16_n4k_workload():
    w = ps.WORKLOADS["bf16_n4k"]
    inp = ps.prefill_inputs(w)
    inp["dO"] = ps.normal((w.B, w.H, w.n, w.d), seed=0, stream=6, dtype="bf16")
    _check(inp, "bf16", w.k, w.pi, w.S, False, "bf16_n4k tc", path="tc")


def test_backward_tensor_core_path_is_deterministic():
    inp = _problem(2, 2, 400, 64, "bf16", seed=5)
    dev = {x: to_dev(inp[x], "bf16") for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    a = [t.clone() for t in pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], 30, 11, 6, path="tc")]
    b = pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], 30, 11, 6, path="tc")
    pia.pi_attn_check()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_gate_gradient_cancels_when_every_key_has_one_prior():
    # S = 0: every key is a window key, log(alpha) shifts every logit alike and cancels, so
    # dLoss/dz = 0 for every row: the oracle's dw_g and db_g are zero up to fp64 rounding and the
    # GPU's within the fp32 rounding bound of the gate gradients (_check)
    (_, _, _, dw, db), (_, _, _, rdw, rdb) = _check(_problem(1, 2, 128, 64, "f32", seed=9), "f32", 16, 32, 0, False,
                                                    "S = 0")
    assert np.max(np.abs(rdw)) < 1e-12 and np.max(np.abs(rdb)) < 1e-12


def test_backward_head_size_256_fp32():
    _check(_problem(1, 1, 90, 256, "f32", seed=3), "f32", 12, 7, 4, False, "d = 256")


def test_backward_bf16_n4k_workload():
    w = ps.WORKLOADS["bf16_n4k"]
    inp = ps.prefill_inputs(w)
    inp["dO"] = ps.normal((w.B, w.H, w.n, w.d), seed=0, stream=6, dtype="bf16")
    _check(inp, "bf16", w.k, w.pi, w.S, False, "bf16_n4k")


def test_backward_is_deterministic():
    inp = _problem(2, 2, 400, 64, "bf16", seed=5)
    dev = {x: to_dev(inp[x], "bf16") for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    a = [t.clone() for t in pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], 30, 11, 6)]
    b = pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], 30, 11, 6)
    pia.pi_attn_check()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("path", ["tc_fused", "tc_split"])
def test_tensor_core_backward_replays_as_a_cuda_graph(path):
    # the tensor-core backward forks its dk/dv passes onto a second stream and joins them back:
    # captured as a CUDA graph on a side stream and replayed, it gives the eager call's bits
    B, H, n, d, k, pi, S = (1, 2, 2560, 64, 50, 10, 20)
    inp = _problem(B, H, n, d, "bf16", seed=41)
    dev = {x: to_dev(inp[x], "bf16") for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    eager = [t.clone() for t in pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], k, pi, S, path=path)]
    pia.pi_attn_check()
    grads = tuple(torch.full_like(t, float("nan")) for t in eager)
    ws = torch.empty(pia.load().pi_attn_bwd_workspace_bytes_ex(B, H, n, d, pia._dtype_code(dev["q"]),
                                                                pia.BWD_PATHS[path]), dtype=torch.uint8, device="cuda")
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
        pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], k, pi, S, grads=grads, workspace=ws,
                        path=path)
    for _ in range(2):
        for t in grads:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        pia.pi_attn_check()
        for name, x, y in zip(("dq", "dk", "dv", "dw_g", "db_g"), eager, grads):
            assert torch.equal(x, y), f"{path}: {name} differs after a graph replay"
    del g
