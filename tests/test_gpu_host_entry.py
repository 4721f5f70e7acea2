"""pi_attn_fwd_host: the prefill over inputs and outputs in host memory, as a pipeline of chunks of
heads (B200 only).

The chunks run the same kernels as pi_attn_fwd_ex on device copies of the same inputs, so out and
lse must be the same bits as a pi_attn_fwd_ex call on the whole problem.  The cases cover chunks
that cross a batch boundary and a ragged last chunk, more chunks than the three rotating buffers
(so every buffer is reused), the split path (its scratch shared by the chunks), the single pass,
the fp32 CUDA-core path, pageable host memory and lse not requested.  One case is also compared
with the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import periodic_sparse_attention_b200 as pia
import pi_synth as ps
from periodic_sparse_attention_b200 import build as pbuild
from tests.gpu_util import assert_close, metrics

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()
    pia.load()
    yield
    torch.cuda.synchronize()


def _host(a, dtype, pinned):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) if dtype == "bf16" \
        else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.pin_memory() if pinned else t.clone()


def _problem(B, H, n, d, dtype, seed):
    return {"q": ps.normal((B, H, n, d), seed=seed, stream=1, dtype=dtype),
            "k": ps.normal((B, H, n, d), seed=seed, stream=2, dtype=dtype),
            "v": ps.normal((B, H, n, d), seed=seed, stream=3, dtype=dtype),
            "w_g": ps.normal((H, d), seed=seed, stream=4, std=d ** -0.5, dtype="f32"),
            "b_g": ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")}


CASES = [  # B, H, n, d, k, pi, S, dtype, path, chunk_heads, pinned, want_lse
    (2, 3, 2048, 128, 100, 64, 12, "bf16", "tc_split", 2, True, True),  # split; chunks 2 + 1 per b
    (1, 8, 4096, 64, 128, 64, 4, "bf16", "tc_fused", 0, True, False),  # single pass, 8 chunks, no lse
    (1, 7, 1000, 64, 40, 100, 5, "bf16", "auto", 1, True, True),       # 7 chunks of one head
    (2, 2, 300, 32, 20, 9, 5, "f32", "auto", 0, False, True),          # CUDA cores, pageable memory
    (1, 4, 2560, 64, 50, 10, 20, "bf16", "tc_split", 3, False, True),  # split, pageable, ragged
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[7]}-{c[8]}-chunk{c[9]}" for c in CASES])
def test_host_entry_gives_the_device_entrys_bits(case):
    B, H, n, d, k, pi, S, dtype, path, chunk, pinned, want_lse = case
    inp = _problem(B, H, n, d, dtype, seed=B * 100 + H + n)
    dev = {x: _host(inp[x], dtype, False).cuda() for x in ("q", "k", "v")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    ref_out, ref_lse = pia.pi_attn_fwd(dev["q"], dev["k"], dev["v"], wg, bg, k, pi, S, path=path)
    host = {x: _host(inp[x], dtype, pinned) for x in ("q", "k", "v")}
    out, lse = pia.pi_attn_fwd_host(host["q"], host["k"], host["v"], wg, bg, k, pi, S, path=path, chunk_heads=chunk,
                                    want_lse=want_lse)
    torch.cuda.synchronize()
    pia.pi_attn_check()
    as_bits = (lambda t: t.view(torch.int16)) if dtype == "bf16" else (lambda t: t.view(torch.int32))
    assert torch.equal(as_bits(out), as_bits(ref_out.cpu())), "out differs from pi_attn_fwd_ex"
    if want_lse:
        assert torch.equal(lse, ref_lse.cpu()), "lse differs from pi_attn_fwd_ex"
    else:
        assert lse is None


def test_host_entry_against_the_oracle_and_back_to_back_calls():
    # two calls in a row on one stream with one workspace: the second must not see the first's
    # buffers (other inputs), and both agree with the fp64 oracle
    B, H, n, d, k, pi, S = 1, 5, 1500, 64, 60, 40, 6
    wsb = pia.pi_attn_fwd_host_workspace_bytes(B, H, n, d, "bf16", 2)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    for seed in (3, 4):
        inp = _problem(B, H, n, d, "bf16", seed)
        wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
        host = {x: _host(inp[x], "bf16", True) for x in ("q", "k", "v")}
        out, lse = pia.pi_attn_fwd_host(host["q"], host["k"], host["v"], wg, bg, k, pi, S, chunk_heads=2, workspace=ws)
        torch.cuda.synchronize()
        pia.pi_attn_check()
        ro, rl, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], k, pi, S)
        got = ps.bf16_bits_to_f32(out.view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
        m = metrics(got.reshape(-1, d), ro.reshape(-1, d), lse.numpy().astype(np.float64).reshape(-1), rl.reshape(-1))
        assert_close(m, "bf16", f"pi_attn_fwd_host, call with seed {seed}")


def test_two_host_threads_share_the_library_streams():
    # the host-buffer prefill and the tensor-core backward use streams and events the library
    # keeps per device; two host threads, each on its own stream with its own problem, call both
    # at once, several times, and each must get its own problem's bits
    import threading
    B, H, n, d, k, pi, S = 1, 4, 2048, 64, 60, 40, 6
    probs = [_problem(B, H, n, d, "bf16", seed) for seed in (21, 22)]
    refs, dev = [], []
    for inp in probs:
        dq = {x: _host(inp[x], "bf16", False).cuda() for x in ("q", "k", "v")}
        wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
        go = torch.from_numpy(ps.normal((B, H, n, d), seed=7, stream=6, dtype="bf16").view(np.int16)).view(
            torch.bfloat16).cuda()
        o, l = pia.pi_attn_fwd(dq["q"], dq["k"], dq["v"], wg, bg, k, pi, S)
        g = pia.pi_attn_bwd(dq["q"], dq["k"], dq["v"], wg, bg, go, k, pi, S, path="tc")
        refs.append((o.cpu(), l.cpu(), [t.cpu() for t in g]))
        dev.append((dq, wg, bg, go, {x: _host(inp[x], "bf16", True) for x in ("q", "k", "v")}))
    torch.cuda.synchronize()
    errors = []

    def work(i):
        try:
            dq, wg, bg, go, host = dev[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(4):
                    out, lse = pia.pi_attn_fwd_host(host["q"], host["k"], host["v"], wg, bg, k, pi, S, chunk_heads=1)
                    g = pia.pi_attn_bwd(dq["q"], dq["k"], dq["v"], wg, bg, go, k, pi, S, path="tc")
                    s.synchronize()
                    ro, rl, rg = refs[i]
                    if not (torch.equal(out.view(torch.int16), ro.view(torch.int16)) and torch.equal(lse, rl)):
                        errors.append(f"thread {i}: host-buffer prefill differs")
                    if not all(torch.equal(a.cpu(), b) for a, b in zip(g, rg)):
                        errors.append(f"thread {i}: backward differs")
        except Exception as e:  # reported below, on the test's thread
            errors.append(f"thread {i}: {e!r}")

    threads = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a thread did not finish"
    pia.pi_attn_check()
    assert not errors, errors


def test_host_entry_replays_as_a_cuda_graph_with_pinned_buffers():
    # captured on a side stream with pinned host buffers (the copy streams join the capture
    # through the call's events) and replayed: the eager call's bits, on the host
    B, H, n, d, k, pi, S = 1, 3, 2048, 64, 60, 40, 6
    inp = _problem(B, H, n, d, "bf16", seed=31)
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    host = {x: _host(inp[x], "bf16", True) for x in ("q", "k", "v")}
    ws = torch.empty(pia.pi_attn_fwd_host_workspace_bytes(B, H, n, d, "bf16", 1), dtype=torch.uint8, device="cuda")
    ref_out, ref_lse = pia.pi_attn_fwd_host(host["q"], host["k"], host["v"], wg, bg, k, pi, S, chunk_heads=1,
                                            workspace=ws)
    torch.cuda.synchronize()
    ref_out, ref_lse = ref_out.clone(), ref_lse.clone()
    out = torch.empty_like(ref_out).pin_memory()
    lse = torch.empty_like(ref_lse).pin_memory()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
        pia.pi_attn_fwd_host(host["q"], host["k"], host["v"], wg, bg, k, pi, S, out=out, lse=lse, chunk_heads=1,
                             workspace=ws)
    for _ in range(2):
        out.view(torch.int16).fill_(-1)
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        pia.pi_attn_check()
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), "out differs after a graph replay"
        assert torch.equal(lse, ref_lse), "lse differs after a graph replay"
    del g


BWD_CASES = [  # B, H, n, d, k, pi, S, dtype, path, bidir, chunk_heads, pinned
    (2, 3, 2048, 64, 100, 64, 12, "bf16", "tc_split", False, 2, True),   # chunks of 2 + 1 heads of both b
    (1, 8, 4096, 64, 128, 64, 4, "bf16", "tc", False, 0, True),          # the bf16_n4k_bwd shape, 8 chunks
    (1, 4, 1024, 64, 40, 32, 6, "bf16", "tc_fused", True, 3, False),     # bidirectional, pageable, ragged
    (2, 2, 300, 32, 20, 9, 5, "f32", "simt", False, 0, True),            # the fp32 CUDA-core backward
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[f"{c[7]}-{c[8]}-bidir{int(c[9])}-chunk{c[10]}" for c in BWD_CASES])
def test_backward_host_entry_gives_the_device_entrys_bits(case):
    B, H, n, d, k, pi, S, dtype, path, bidir, chunk, pinned = case
    inp = _problem(B, H, n, d, dtype, seed=7 * H + n)
    inp["dO"] = ps.normal((B, H, n, d), seed=5, stream=6, dtype=dtype)
    dev = {x: _host(inp[x], dtype, False).cuda() for x in ("q", "k", "v", "dO")}
    wg, bg = torch.from_numpy(inp["w_g"]).cuda(), torch.from_numpy(inp["b_g"]).cuda()
    ref = [t.cpu() for t in pia.pi_attn_bwd(dev["q"], dev["k"], dev["v"], wg, bg, dev["dO"], k, pi, S, bidir=bidir,
                                             path=path)]
    host = {x: _host(inp[x], dtype, pinned) for x in ("q", "k", "v", "dO")}
    got = pia.pi_attn_bwd_host(host["q"], host["k"], host["v"], wg, bg, host["dO"], k, pi, S, bidir=bidir, path=path,
                               chunk_heads=chunk)
    torch.cuda.synchronize()
    pia.pi_attn_check()
    for name, x, y in zip(("dq", "dk", "dv", "dw_g", "db_g"), got, ref):
        assert torch.equal(x.cpu(), y), f"{name} differs from pi_attn_bwd_ex"
