"""The compact ring cache on the GPU: decode over it (pi_attn_decode_ring) and the constant-time
update (pi_attn_cache_append), against the fp64 decode oracle on the full cache (B200 only).

A ring of capacity C keeps position j in slot j mod C.  The tests fill it from a full-length
cache, or token by token through the append, starting from a ring of NaN so that a read of a slot
that was never written (or was already overwritten) shows in the output.
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


def _full(B, H, n, d, seed):
    q = ps.normal((B, H, n, d), seed=seed, stream=1, dtype="bf16")  # q of every position (decode uses one)
    k = ps.normal((B, H, n, d), seed=seed, stream=2, dtype="bf16")
    v = ps.normal((B, H, n, d), seed=seed, stream=3, dtype="bf16")
    w_g = ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")
    return q, k, v, w_g, b_g


def _nan_ring(B, H, C, d):
    r = torch.empty((B, H, C, d), dtype=torch.bfloat16, device="cuda")
    r.view(torch.int16).fill_(-1)  # all bits set: NaN
    return r


def _oracle_step(q, k, v, w_g, b_g, lengths, kw, pi, S):
    B, H = q.shape[:2]
    qd = np.stack([q[b, :, lengths[b] - 1] for b in range(B)])
    return oracle.decode(qd, k, v, w_g, b_g, kw, pi, S, lengths=np.asarray(lengths, np.int32))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("extra", [0, 19])  # capacity = max(k, S pi) + 1 + extra
@pytest.mark.parametrize("shape", [
    (2, 3, 40, 16, 5),    # one CTA per (b, h)
    (1, 2, 300, 64, 7),   # few (b, h) and k + 1 + S > 128: each (b, h) split across CTAs, then merged
])
def test_ring_decode_matches_full_cache_oracle(d, extra, shape):
    B, H, kw, pi, S = shape
    C = max(kw, S * pi) + 1 + extra
    lengths = [1500, C - 3][:B]  # one sequence wrapped several times, one not yet wrapped
    n = max(lengths)
    q, k, v, w_g, b_g = _full(B, H, n, d, seed=d + extra)
    kr, vr = _nan_ring(B, H, C, d), _nan_ring(B, H, C, d)
    kt, vt = to_dev(k, "bf16"), to_dev(v, "bf16")
    for b, L in enumerate(lengths):
        for pos in range(max(0, L - C), L):  # the last C positions of each sequence
            kr[b, :, pos % C] = kt[b, :, pos]
            vr[b, :, pos % C] = vt[b, :, pos]
    qd = torch.stack([to_dev(q[b, :, L - 1], "bf16") for b, L in enumerate(lengths)])
    cl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out, lse = pia.pi_attn_decode_ring(qd, kr, vr, torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda(), cl, kw,
                                       pi, S)
    pia.pi_attn_check()
    ro, rl, _ = _oracle_step(q, k, v, w_g, b_g, lengths, kw, pi, S)
    assert_close(metrics(from_dev(out).reshape(B * H, d), ro, lse.cpu().numpy().astype(np.float64).reshape(-1), rl),
                 "bf16", f"ring d={d} C={C}")


def test_append_token_by_token_then_decode():
    B, H, d, kw, pi, S = 2, 2, 64, 12, 8, 4
    C = max(kw, S * pi) + 1
    T = 3 * C + 5
    q, k, v, w_g, b_g = _full(B, H, T, d, seed=77)
    kt, vt = to_dev(k, "bf16"), to_dev(v, "bf16")
    kr, vr = _nan_ring(B, H, C, d), _nan_ring(B, H, C, d)
    cl = torch.zeros(B, dtype=torch.int32, device="cuda")
    wg, bg = torch.from_numpy(w_g).cuda(), torch.from_numpy(b_g).cuda()
    checks = {1, C - 1, C, C + 1, 2 * C + 3, T}
    for step in range(1, T + 1):
        pos = step - 1
        pia.pi_attn_cache_append(kr, vr, kt[:, :, pos].contiguous(), vt[:, :, pos].contiguous(), cl)
        if step in checks:
            qd = to_dev(np.ascontiguousarray(q[:, :, pos]), "bf16")
            out, lse = pia.pi_attn_decode_ring(qd, kr, vr, wg, bg, cl, kw, pi, S)
            pia.pi_attn_check()
            assert cl.cpu().tolist() == [step] * B
            ro, rl, _ = _oracle_step(q, k, v, w_g, b_g, [step] * B, kw, pi, S)
            assert_close(metrics(from_dev(out).reshape(B * H, d), ro, lse.cpu().numpy().astype(np.float64).reshape(-1),
                                 rl), "bf16", f"append step {step}")
    # the ring holds exactly the last C positions, each in its slot
    for pos in range(T - C, T):
        assert torch.equal(kr[:, :, pos % C].view(torch.int16), kt[:, :, pos].view(torch.int16))
        assert torch.equal(vr[:, :, pos % C].view(torch.int16), vt[:, :, pos].view(torch.int16))
