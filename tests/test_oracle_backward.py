"""The backward oracle (gradients through out) pinned against things other than itself (CPU only).

  * central finite differences of the forward oracle (itself pinned by test_oracle_pins.py): every
    input element of a small problem, causal and bidirectional
  * torch autograd through a dense float64 formulation of the operator (masks from brute.masks,
    the gate as log-sigmoid priors, softmax, P V): an independent statement whose gradient is the
    library's, not a retyped formula
The mistakes they are there to catch: a dropped gate term in dq, a wrong sign or factor on the
priors' derivatives (1 - alpha, -alpha), a missing tau, dv built from ds instead of p, D_i left out.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.brute as brute
import pi_synth as ps


def _problem(B, H, n, d, seed):
    q = ps.normal((B, H, n, d), seed=seed, stream=1, dtype="f32")
    k = ps.normal((B, H, n, d), seed=seed, stream=2, dtype="f32")
    v = ps.normal((B, H, n, d), seed=seed, stream=3, dtype="f32")
    w_g = ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")
    G = ps.normal((B, H, n, d), seed=seed, stream=6, dtype="f32").astype(np.float64)  # dLoss/dout
    return q, k, v, w_g, b_g, G


def _loss(q, k, v, w_g, b_g, G, kwin, pi, S, bidir):
    out, _, _ = oracle.fwd(q, k, v, w_g, b_g, kwin, pi, S, bidir=bidir, nthreads=1)
    return float(np.sum(out * G))


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("n,kwin,pi,S", [(12, 3, 4, 2), (10, 1, 2, 4)])
def test_backward_matches_finite_differences(n, kwin, pi, S, bidir):
    B, H, d = 1, 2, 4
    q, k, v, w_g, b_g, G = _problem(B, H, n, d, seed=n * 3 + kwin)
    grads = dict(zip(["q", "k", "v", "w_g", "b_g"], oracle.bwd(q, k, v, w_g, b_g, G, kwin, pi, S, bidir=bidir)))
    args = {"q": q, "k": k, "v": v, "w_g": w_g, "b_g": b_g}
    h = np.float32(2.0 ** -8)
    for name, arr in args.items():
        flat = arr.reshape(-1)
        g = grads[name].reshape(-1)
        for e in range(flat.size):
            keep = flat[e]
            flat[e] = np.float32(keep + h)
            xp = float(flat[e])
            lp = _loss(q, k, v, w_g, b_g, G, kwin, pi, S, bidir)
            flat[e] = np.float32(keep - h)
            xm = float(flat[e])
            lm = _loss(q, k, v, w_g, b_g, G, kwin, pi, S, bidir)
            flat[e] = keep
            fd = (lp - lm) / (xp - xm)
            assert abs(fd - g[e]) <= 2e-4 * max(1.0, abs(fd)), (name, e, fd, g[e])


def _dense_torch(q, k, v, w_g, b_g, kwin, pi, S, bidir):
    n, d = q.shape[2], q.shape[3]
    W, P = (torch.from_numpy(m) for m in brute.masks(n, kwin, pi, S, bidir))
    z = torch.einsum("bhnd,hd->bhn", q, w_g) + b_g[None, :, None]
    log_a = torch.nn.functional.logsigmoid(z)[..., None]
    log_1ma = torch.nn.functional.logsigmoid(-z)[..., None]
    bias = torch.where(W, log_a, torch.where(P, log_1ma, torch.tensor(float("-inf"), dtype=torch.float64)))
    scores = torch.einsum("bhid,bhjd->bhij", q, k) / math.sqrt(d) + bias
    return torch.einsum("bhij,bhjd->bhid", torch.softmax(scores, dim=-1), v)


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("n,kwin,pi,S,d", [(40, 5, 7, 4, 8), (33, 0, 1, 12, 4), (48, 16, 8, 3, 16), (20, 30, 3, 5, 8)])
def test_backward_matches_torch_autograd(n, kwin, pi, S, d, bidir):
    B, H = 2, 2
    q, k, v, w_g, b_g, G = _problem(B, H, n, d, seed=n + 11 * kwin)
    leaves = [torch.tensor(x.astype(np.float64), requires_grad=True) for x in (q, k, v, w_g, b_g)]
    out = _dense_torch(*leaves, kwin, pi, S, bidir)
    (out * torch.from_numpy(G)).sum().backward()
    got = oracle.bwd(q, k, v, w_g, b_g, G, kwin, pi, S, bidir=bidir)
    for name, ref, g in zip(["dq", "dk", "dv", "dw_g", "db_g"], leaves, got):
        np.testing.assert_allclose(g, ref.grad.numpy(), rtol=0, atol=1e-11, err_msg=name)


@pytest.mark.parametrize("bidir", [False, True])
def test_gate_gradient_is_zero_when_one_prior_covers_every_key(bidir):
    # with S = 0 every key of a row carries log(alpha): the prior shifts all logits alike and cancels
    # in the softmax, so dLoss/dz = (1 - alpha) sum_j ds_j = (1 - alpha) (D - D) = 0
    q, k, v, w_g, b_g, G = _problem(2, 3, 40, 8, seed=31)
    _, _, _, dw, db = oracle.bwd(q, k, v, w_g, b_g, G, 6, 5, 0, bidir=bidir)
    assert np.max(np.abs(dw)) < 1e-12 and np.max(np.abs(db)) < 1e-12
    # and it does not vanish once skips are present
    _, _, _, dw2, db2 = oracle.bwd(q, k, v, w_g, b_g, G, 6, 5, 4, bidir=bidir)
    assert np.max(np.abs(db2)) > 1e-3


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("n,kwin,pi,S,d", [(64, 8, 16, 3, 8), (300, 20, 9, 5, 16), (129, 0, 1, 40, 4)])
def test_key_and_value_gradients_sum_to_their_closed_forms(n, kwin, pi, S, d, bidir):
    # Each row's weights p_ij sum to one over its keys, so sum_j dv_j = sum_j sum_i p_ij dO_i =
    # sum_i dO_i; and each row's ds_ij = p_ij (dp_ij - D_i) sums to D_i - D_i = 0 whatever the gate's
    # priors, so sum_j dk_j = tau sum_i q_i sum_j ds_ij = 0.  Both hold per (b, h) and column; a
    # dropped key, a weight counted twice or a wrong D breaks them.
    q, k, v, w_g, b_g, G = _problem(2, 2, n, d, seed=n + S)
    _, dk, dv, _, _ = oracle.bwd(q, k, v, w_g, b_g, G, kwin, pi, S, bidir=bidir)
    scale_v = np.linalg.norm(G, axis=2)
    np.testing.assert_allclose(dv.sum(axis=2), G.sum(axis=2), rtol=0, atol=1e-12 * scale_v.max())
    scale_k = np.linalg.norm(dk, axis=2)
    assert np.max(np.abs(dk.sum(axis=2)) / scale_k) < 1e-12
