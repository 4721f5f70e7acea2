"""CUDA path against the fp64 oracle, element by element, through the C ABI (B200 only).

Small cases compare every row; the full-size workloads compare sampled rows (4096 random query
rows plus the boundary rows of every (b, h)) in the same launch configuration the bench times.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from tests.gpu_util import assert_close, from_dev, metrics, sampled_rows, to_dev

pytestmark = pytest.mark.gpu

TC = "tc"


@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()
    pia.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()


def _tc_applies(dtype, d):
    return dtype == "bf16" and d in (64, 128)


def _dev_inputs(inp, dtype):
    return (to_dev(inp["q"], dtype), to_dev(inp["k"], dtype), to_dev(inp["v"], dtype),
            torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda())


def _run_fwd(inp, dtype, k, pi, S, path="auto"):
    q, kk, v, wg, bg = _dev_inputs(inp, dtype)
    out, lse = pia.pi_attn_fwd(q, kk, v, wg, bg, k, pi, S, path=path)
    pia.pi_attn_check()
    return from_dev(out), lse.cpu().numpy().astype(np.float64)


def _inputs(B, H, n, d, dtype, seed, bg_std=0.7):
    q = ps.normal((B, H, n, d), seed=seed, stream=1, dtype=dtype)
    k = ps.normal((B, H, n, d), seed=seed, stream=2, dtype=dtype)
    v = ps.normal((B, H, n, d), seed=seed, stream=3, dtype=dtype)
    w_g = ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=5, std=bg_std, dtype="f32")
    return {"q": q, "k": k, "v": v, "w_g": w_g, "b_g": b_g}


# ------------------------------------------------------------------------------------------------
# the workloads
# ------------------------------------------------------------------------------------------------

def test_tiny_f32_every_row():
    w = ps.WORKLOADS["tiny_f32"]
    inp = ps.prefill_inputs(w)
    out, lse = _run_fwd(inp, "f32", w.k, w.pi, w.S)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], w.k, w.pi, w.S)
    assert_close(metrics(out, ro, lse, rl), "f32", "tiny_f32")


@pytest.mark.parametrize("path", ["auto", "simt", TC, "tc_fused", "tc_split"])
def test_bf16_n4k_every_row(path):
    w = ps.WORKLOADS["bf16_n4k"]
    inp = ps.prefill_inputs(w)
    out, lse = _run_fwd(inp, "bf16", w.k, w.pi, w.S, path)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], w.k, w.pi, w.S)
    assert_close(metrics(out, ro, lse, rl), "bf16", f"bf16_n4k/{path}")


@pytest.mark.parametrize("path", ["auto", "tc_fused", "tc_split"])
@pytest.mark.parametrize("name", ["bf16_n32k", "bf16_n128k"])
def test_long_workloads_sampled_rows(name, path):
    w = ps.WORKLOADS[name]
    inp = ps.prefill_inputs(w)
    out, lse = _run_fwd(inp, "bf16", w.k, w.pi, w.S, path)
    rows = sampled_rows(w, 4096)
    ro, rl, _ = oracle.fwd_rows(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], w.k, w.pi, w.S, rows=rows)
    m = metrics(out.reshape(-1, w.d)[rows], ro, lse.reshape(-1)[rows], rl)
    assert_close(m, "bf16", name)
    # properties that hold at every row, checked on all of them
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def test_decode_workload_full_cache():
    w = ps.WORKLOADS["decode_bf16"]
    inp = ps.decode_inputs(w)
    B, H, n, d = w.B, w.H, w.n, w.d
    pos = torch.from_numpy(inp["pos"]).cuda()
    kc = torch.empty((B, H, n, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    kc.view(torch.int16).fill_(-1)  # all bits set: NaN, so a stray read shows in the output
    vc.view(torch.int16).fill_(-1)
    kc[:, :, pos] = to_dev(inp["kc"], "bf16")
    vc[:, :, pos] = to_dev(inp["vc"], "bf16")
    q = to_dev(inp["q"], "bf16")
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    out, lse = pia.pi_attn_decode(q, kc, vc, wg, bg, w.k, w.pi, w.S)
    pia.pi_attn_check()
    out, lse = from_dev(out), lse.cpu().numpy().astype(np.float64)
    del kc, vc
    torch.cuda.empty_cache()
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    rng = np.random.default_rng(0)
    pick = np.unique(np.concatenate([rng.choice(B * H, 48, replace=False), [0, B * H - 1]]))
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for bh in pick:
        b, h = divmod(int(bh), H)
        ks = np.full((1, 1, n, d), 0xFFFF, dtype=np.uint16)
        vs = np.full((1, 1, n, d), 0xFFFF, dtype=np.uint16)
        ks[0, 0, inp["pos"]] = inp["kc"][b, h]
        vs[0, 0, inp["pos"]] = inp["vc"][b, h]
        o, l, _ = oracle.decode(inp["q"][b, h][None, None], ks, vs, inp["w_g"][h][None], inp["b_g"][h][None], w.k,
                                w.pi, w.S)
        ref_o.append(o[0]), ref_l.append(l[0]), got_o.append(out[b, h]), got_l.append(lse[b, h])
    assert_close(metrics(np.array(got_o), np.array(ref_o), np.array(got_l), np.array(ref_l)), "bf16", "decode")


# ------------------------------------------------------------------------------------------------
# edge cases: tiny, ragged, degenerate
# ------------------------------------------------------------------------------------------------

EDGE = [  # B, H, n, d, k, pi, S
    (1, 1, 1, 64, 0, 1, 1),        # a single token
    (2, 3, 1000, 128, 100, 37, 12),  # ragged tail, many skips
    (1, 2, 333, 64, 400, 16, 40),   # window longer than the sequence
    (1, 1, 200, 128, 64, 32, 0),    # no skips: causal sliding window
    (1, 1, 300, 64, 8, 1, 50),      # period 1
    (1, 2, 513, 128, 128, 64, 6),   # ties m*pi == k
    (1, 1, 130, 64, 5, 7, 3),       # tiny window, ragged
    (2, 2, 640, 128, 0, 128, 4),    # window of the token alone
    (1, 1, 385, 64, 127, 129, 2),   # window just under a tile, period just over
    (1, 2, 1024, 128, 64, 256, 3),  # residue sequences of 4 rows
    (2, 1, 2048, 64, 100, 128, 8),  # residue sequences of 16 rows, first skip m = 1
    (1, 1, 4096, 128, 300, 256, 12),  # first surviving skip m = 2
    (1, 1, 2112, 64, 10, 64, 40),   # 33 rows per residue, skips reach the start
    (1, 2, 100, 64, 8, 200, 3),     # period longer than the sequence: no skip exists
    (1, 1, 2100, 128, 513, 300, 7),  # window not a multiple of a key tile; last 256-row block ragged
    (3, 5, 768, 128, 1000, 128, 9),  # window longer than the sequence: the skips of m >= 8 lie before it
]


def _split_applies(n, k, pi, S):
    # the forward's split: at least one whole period (the residue view), a skip outside the window
    return n >= pi and S >= k // pi + 1


@pytest.mark.parametrize("path", ["auto", "simt", TC, "tc_fused", "tc_split"])
@pytest.mark.parametrize("case", EDGE)
def test_edge_cases_bf16(case, path):
    B, H, n, d, k, pi, S = case
    inp = _inputs(B, H, n, d, "bf16", seed=n + 7 * k)
    if path.startswith("tc") and not _tc_applies("bf16", d):
        pytest.skip("tensor-core path does not cover this head size")
    if path == "tc_split" and not _split_applies(n, k, pi, S):
        pytest.skip("split path needs n >= pi and a skip outside the window")
    out, lse = _run_fwd(inp, "bf16", k, pi, S, path)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S)
    assert_close(metrics(out, ro, lse, rl), "bf16", f"{case}/{path}")


@pytest.mark.parametrize("case", [(1, 1, 1, 32, 0, 1, 1), (2, 3, 257, 32, 8, 16, 2), (1, 2, 300, 128, 40, 9, 7),
                                  (1, 1, 100, 4, 3, 2, 5), (1, 1, 70, 256, 30, 20, 3)])
def test_edge_cases_f32(case):
    B, H, n, d, k, pi, S = case
    inp = _inputs(B, H, n, d, "f32", seed=n + k)
    out, lse = _run_fwd(inp, "f32", k, pi, S)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S)
    assert_close(metrics(out, ro, lse, rl), "f32", str(case))


@pytest.mark.parametrize("path", ["auto", "simt", "tc_fused", "tc_split"])
@pytest.mark.parametrize("bias", [60.0, -60.0])
def test_gate_saturation(bias, path):
    B, H, n, d, k, pi, S = 1, 2, 768, 128, 64, 96, 6
    inp = _inputs(B, H, n, d, "bf16", seed=11)
    inp["w_g"][:] = 0
    inp["b_g"][:] = bias
    out, lse = _run_fwd(inp, "bf16", k, pi, S, path)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S)
    assert_close(metrics(out, ro, lse, rl), "bf16", f"bias {bias}/{path}")


@pytest.mark.parametrize("path", ["auto", "simt", "tc_fused", "tc_split"])
def test_rows_are_normalised(path):
    # V = 1 everywhere: every output element must be 1 (the weights of each row sum to one)
    inp = _inputs(1, 4, 1280, 128, "bf16", seed=3)
    inp["v"][:] = 0x3F80  # bf16 1.0
    out, _ = _run_fwd(inp, "bf16", 256, 256, 8, path)
    assert np.max(np.abs(out - 1.0)) <= 4e-3


def test_split_workspace_from_caller_or_library_gives_identical_results():
    # pi_attn_fwd_ex allocates the skip partials itself; the binding passes a torch workspace to
    # pi_attn_fwd_ws.  Same kernels, same scratch layout: the results are bit-identical.
    import ctypes
    inp = _inputs(2, 3, 2048, 64, "bf16", seed=9)
    q, kk, v, wg, bg = _dev_inputs(inp, "bf16")
    out_ws, lse_ws = pia.pi_attn_fwd(q, kk, v, wg, bg, 100, 128, 9, path="tc_split")
    out_lib, lse_lib = torch.empty_like(q), torch.empty_like(lse_ws)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = pia.load().pi_attn_fwd_ex(p(q), p(kk), p(v), p(wg), p(bg), p(out_lib), p(lse_lib), 2, 3, 2048, 64, 100, 128, 9,
                                   pia.PI_ATTN_BF16, pia.PATHS["tc_split"],
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pia.PI_ATTN_OK
    pia.pi_attn_check()
    assert torch.equal(out_ws.view(torch.int16), out_lib.view(torch.int16))
    assert torch.equal(lse_ws, lse_lib)
    ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], 100, 128, 9)
    assert_close(metrics(from_dev(out_ws).reshape(-1, 64), ro.reshape(-1, 64), lse_ws.cpu().numpy().reshape(-1),
                         rl.reshape(-1)), "bf16", "split path, caller workspace")


def test_lse_is_optional():
    inp = _inputs(1, 1, 300, 64, "bf16", seed=5)
    q, kk, v, wg, bg = _dev_inputs(inp, "bf16")
    out, lse = pia.pi_attn_fwd(q, kk, v, wg, bg, 16, 8, 3, want_lse=False)
    pia.pi_attn_check()
    assert lse is None
    ro, _, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], 16, 8, 3)
    assert np.max(np.abs(from_dev(out) - ro)) <= 2e-2


@pytest.mark.parametrize("n,k,pi,S", [(1000, 8, 16, 2), (4096, 128, 64, 4), (3000, 256, 256, 8), (777, 0, 1, 70),
                                      (500, 600, 7, 3), (300, 20, 5, 0)])
def test_index_sets_bit_exact(n, k, pi, S):
    c, idx = pia.pi_attn_debug_index_sets(n, k, pi, S)
    torch.cuda.synchronize()
    rc, ridx = oracle.index_table(n, k, pi, S)
    assert np.array_equal(c.cpu().numpy(), rc)
    assert np.array_equal(idx.cpu().numpy(), ridx)


# ------------------------------------------------------------------------------------------------
# decode variants
# ------------------------------------------------------------------------------------------------

def _decode_case(B, H, n_cache, d, k, pi, S, dtype, lengths, seed=0):
    q = ps.normal((B, H, d), seed=seed, stream=11, dtype=dtype)
    kc = ps.normal((B, H, n_cache, d), seed=seed, stream=12, dtype=dtype)
    vc = ps.normal((B, H, n_cache, d), seed=seed, stream=13, dtype=dtype)
    w_g = ps.normal((H, d), seed=seed, stream=14, std=1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=15, std=0.7, dtype="f32")
    cl = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out, lse = pia.pi_attn_decode(to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype), torch.from_numpy(w_g).cuda(),
                                  torch.from_numpy(b_g).cuda(), k, pi, S, cache_len=cl)
    return q, kc, vc, w_g, b_g, out, lse


@pytest.mark.parametrize("case", [
    (3, 2, 700, 128, 64, 50, 9, "bf16", [700, 1, 333]),
    (2, 3, 5000, 64, 1024, 97, 31, "bf16", None),
    (1, 2, 9000, 128, 1024, 2048, 31, "bf16", [8999]),   # few (b, h): split path
    (1, 1, 70000, 64, 4000, 700, 60, "bf16", None),      # split path, d = 64
    (2, 2, 300, 32, 20, 9, 5, "f32", [300, 17]),         # fp32 decode
    (2, 1, 400, 96, 30, 11, 4, "bf16", [400, 2]),        # bf16 head size without the fast kernel
])
def test_decode_variants(case):
    B, H, n_cache, d, k, pi, S, dtype, lengths = case
    q, kc, vc, w_g, b_g, out, lse = _decode_case(B, H, n_cache, d, k, pi, S, dtype, lengths)
    pia.pi_attn_check()
    ro, rl, _ = oracle.decode(q, kc, vc, w_g, b_g, k, pi, S, lengths=lengths)
    assert_close(metrics(from_dev(out).reshape(B * H, d), ro, lse.cpu().numpy().reshape(-1), rl), dtype, str(case))


def test_decode_rejects_bad_cache_length_on_device():
    B, H, n_cache, d = 2, 2, 64, 128
    _, _, _, _, _, out, lse = _decode_case(B, H, n_cache, d, 8, 4, 3, "bf16", [0, 65])
    with pytest.raises(pia.PiAttnError) as e:
        pia.pi_attn_check()
    assert e.value.status == pia.PI_ATTN_EDEVICE
    assert torch.isnan(out.float()).all() and torch.isnan(lse).all()
    pia.pi_attn_check()  # the word was cleared by the first check
