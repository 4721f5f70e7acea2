"""The fp64 oracle pinned against things other than itself (CPU only).

Pins, and the mistake each one is there to catch:
  * the worked mask example of the "Sliding Window Attention" page (58 vs 136 scores, reach
    4/7/10/13)                                   -> window extent / off-by-one in L(i)
  * closed-form totals of |L| and |P|            -> skip de-duplication rule, sequence-start rule
  * brute-force set enumeration (dense masks)    -> any index error, ties m*pi == k
  * dense brute force and torch SDPA with the bias as attn_mask -> transposed operands, scale,
                                                    softmax / lse mistakes
  * closed forms with q = 0 and with k = 0       -> gate sign, gate on scaled vs unscaled q,
                                                    prior scaled by tau, natural vs base-2 lse
  * alpha -> 1 (and S = 0) equals causal sliding-window attention; alpha -> 0 equals
    skip-only attention                           -> which prior goes with which set
  * rows sum to 1; decode equals the last prefill row
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.brute as brute
import pi_synth as ps


def _inputs(B, H, n, d, seed, dtype="bf16", wg_std=None, bg_std=0.7):
    q = ps.normal((B, H, n, d), seed=seed, stream=1, dtype=dtype)
    k = ps.normal((B, H, n, d), seed=seed, stream=2, dtype=dtype)
    v = ps.normal((B, H, n, d), seed=seed, stream=3, dtype=dtype)
    w_g = ps.normal((H, d), seed=seed, stream=4, std=wg_std or 1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=5, std=bg_std, dtype="f32")
    return q, k, v, w_g, b_g


# ----------------------------------------------------------------------------------------------
# index rule
# ----------------------------------------------------------------------------------------------

def test_page_worked_example_score_counts(golden):
    g = golden("swa_worked_example.txt")
    n = int(g["seq_len"][0])
    k = int(g["page_window"][0]) - 1  # the page's window counts the token itself
    assert oracle.counts(n, k, 5, 0) == (int(g["scores_window"][0]), 0)
    assert oracle.counts(n, n - 1, 5, 0) == (int(g["scores_full_causal"][0]), 0)
    assert oracle.counts(n, 10 * n, 5, 0) == (int(g["scores_full_causal"][0]), 0)


def test_page_worked_example_reach(golden):
    g = golden("swa_worked_example.txt")
    n = int(g["seq_len"][0])
    k = int(g["page_window"][0]) - 1
    cnt, idx = oracle.index_table(n, k, 5, 0)
    A = np.zeros((n, n), dtype=np.int64)
    for i in range(n):
        for j in idx[i, : cnt[i, 0]]:
            A[i, j] = 1
    reach = A > 0
    got = []
    for _ in range(4):
        got.append(int(reach[-1].sum()))
        reach = (A @ reach.astype(np.int64)) > 0
    assert got == [int(x) for x in g["reach_by_layer"]]


def _closed_form_totals(n, k, pi, S):
    # sum_i (min(i, k) + 1)
    if n <= k + 1:
        sl = n * (n + 1) // 2
    else:
        sl = (k + 1) * (k + 2) // 2 + (n - k - 1) * (k + 1)
    # a skip m survives when m*pi > k; it exists for the n - m*pi rows i >= m*pi
    m0 = k // pi + 1
    sp = sum(max(0, n - m * pi) for m in range(m0, S + 1))
    return sl, sp


@pytest.mark.parametrize("n,k,pi,S", [
    (256, 8, 16, 2), (4096, 128, 64, 4), (32768, 256, 256, 8), (131072, 512, 1024, 16),
    (65536, 1024, 2048, 31), (16, 3, 4, 5), (100, 12, 4, 9), (100, 12, 3, 4), (57, 0, 1, 60), (5, 9, 2, 3),
    (1, 0, 1, 1), (300, 64, 32, 2),
])
def test_index_totals_closed_form(n, k, pi, S):
    assert oracle.counts(n, k, pi, S) == _closed_form_totals(n, k, pi, S)


@pytest.mark.parametrize("n,k,pi,S", [
    (32, 3, 4, 5), (40, 8, 4, 6), (48, 5, 7, 9), (33, 0, 1, 40), (64, 16, 8, 4), (64, 16, 16, 3),
    (20, 6, 3, 10), (64, 63, 2, 40), (17, 4, 5, 0),
])
def test_index_sets_match_dense_masks(n, k, pi, S):
    W, P = brute.masks(n, k, pi, S)
    for i in range(n):
        L_o, P_o = oracle.index_set(i, k, pi, S)
        assert L_o.tolist() == np.nonzero(W[i])[0].tolist()
        assert sorted(P_o.tolist()) == np.nonzero(P[i])[0].tolist()
        assert not set(L_o.tolist()) & set(P_o.tolist())
        # P by increasing m means decreasing key index
        assert P_o.tolist() == sorted(P_o.tolist(), reverse=True)


def test_index_table_layout():
    cnt, idx = oracle.index_table(40, 4, 3, 6, width=4 + 1 + 6)
    for i in [0, 3, 4, 5, 17, 39]:
        L_o, P_o = oracle.index_set(i, 4, 3, 6)
        assert cnt[i].tolist() == [L_o.size, P_o.size]
        row = idx[i].tolist()
        assert row[: L_o.size + P_o.size] == L_o.tolist() + P_o.tolist()
        assert all(x == -1 for x in row[L_o.size + P_o.size:])


# ----------------------------------------------------------------------------------------------
# attention core
# ----------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n,k,pi,S,d", [
    (32, 3, 4, 5, 16), (48, 5, 7, 9, 8), (33, 0, 1, 40, 16), (64, 16, 8, 4, 32), (64, 16, 16, 3, 12),
    (20, 6, 3, 10, 4), (1, 0, 1, 1, 8), (7, 2, 9, 3, 16),
])
def test_oracle_matches_dense_brute_force(dtype, n, k, pi, S, d):
    q, kk, v, w_g, b_g = _inputs(2, 3, n, d, seed=n * 31 + k, dtype=dtype)
    out, lse, rs = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S)
    out_b, lse_b, _ = brute.attention(q, kk, v, w_g, b_g, k, pi, S)
    np.testing.assert_allclose(out, out_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(rs, 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n,k,pi,S,d", [(40, 6, 5, 7, 16), (64, 9, 3, 30, 32)])
def test_brute_force_matches_torch_sdpa(n, k, pi, S, d):
    q, kk, v, w_g, b_g = _inputs(1, 2, n, d, seed=7)
    out_b, lse_b, bias = brute.attention(q, kk, v, w_g, b_g, k, pi, S)
    tq, tk, tv = (torch.from_numpy(brute.widen(x)) for x in (q, kk, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(bias))
    np.testing.assert_allclose(out_b, ref.numpy(), rtol=0, atol=1e-12)
    # the oracle against the library routine directly
    out, lse, _ = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    scores = torch.einsum("bhid,bhjd->bhij", tq, tk) / math.sqrt(d) + torch.from_numpy(bias)
    np.testing.assert_allclose(lse, torch.logsumexp(scores, dim=-1).numpy(), rtol=0, atol=1e-12)


def _set_sizes(n, k, pi, S):
    W, P = brute.masks(n, k, pi, S)
    return W, P, W.sum(1).astype(np.float64), P.sum(1).astype(np.float64)


def test_gate_closed_form_zero_query():
    # q = 0: every logit is just its prior, z = b_g, alpha = sigmoid(b_g).
    n, k, pi, S, d, H = 60, 5, 4, 9, 16, 3
    q, kk, v, w_g, b_g = _inputs(1, H, n, d, seed=3, dtype="f32", bg_std=1.5)
    q = np.zeros_like(q)
    out, lse, _ = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S)
    W, P, nL, nP = _set_sizes(n, k, pi, S)
    vd = v.astype(np.float64)
    for h in range(H):
        a = 1.0 / (1.0 + math.exp(-float(b_g[h])))
        den = a * nL + (1 - a) * nP
        np.testing.assert_allclose(lse[0, h], np.log(den), rtol=0, atol=1e-12)
        num = a * (W.astype(np.float64) @ vd[0, h]) + (1 - a) * (P.astype(np.float64) @ vd[0, h])
        np.testing.assert_allclose(out[0, h], num / den[:, None], rtol=0, atol=1e-12)


def test_gate_closed_form_zero_keys():
    # k = 0: every dot product vanishes, so only the gate remains; alpha uses the UNSCALED query.
    n, k, pi, S, d, H = 50, 3, 6, 7, 32, 2
    q, kk, v, w_g, b_g = _inputs(1, H, n, d, seed=4, dtype="f32", wg_std=0.5)
    kk = np.zeros_like(kk)
    out, lse, _ = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S)
    W, P, nL, nP = _set_sizes(n, k, pi, S)
    for h in range(H):
        z = q[0, h].astype(np.float64) @ w_g[h].astype(np.float64) + float(b_g[h])
        a = 1.0 / (1.0 + np.exp(-z))
        den = a * nL + (1 - a) * nP
        np.testing.assert_allclose(lse[0, h], np.log(den), rtol=0, atol=1e-12)
        num = a[:, None] * (W.astype(np.float64) @ v[0, h]) + (1 - a)[:, None] * (P.astype(np.float64) @ v[0, h])
        np.testing.assert_allclose(out[0, h], num / den[:, None], rtol=0, atol=1e-12)


def _sdpa_masked(q, k, v, mask):
    tq, tk, tv = (torch.from_numpy(brute.widen(x)) for x in (q, k, v))
    m = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m)
    s = torch.einsum("bhid,bhjd->bhij", tq, tk) / math.sqrt(q.shape[-1])
    s = s.masked_fill(~m, float("-inf"))
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


def test_alpha_to_one_is_causal_sliding_window():
    # S = 0: exactly causal sliding-window attention; the page's own mask construction
    # (offset >= 0) & (offset < window) with window = k + 1, through the library routine.
    n, k, d = 64, 6, 16
    q, kk, v, w_g, b_g = _inputs(1, 2, n, d, seed=5)
    pos = np.arange(n)
    off = pos[:, None] - pos[None, :]
    swa = (off >= 0) & (off < k + 1)
    o_ref, lse_ref = _sdpa_masked(q, kk, v, swa)
    out, lse, _ = oracle.fwd(q, kk, v, w_g, b_g, k, 4, 0)
    np.testing.assert_allclose(out, o_ref, rtol=0, atol=1e-12)
    # the prior log(alpha) shifts lse only
    z = np.einsum("bhnd,hd->bhn", brute.widen(q), w_g.astype(np.float64)) + b_g[None, :, None]
    np.testing.assert_allclose(lse - (-np.log1p(np.exp(-z))), lse_ref, rtol=0, atol=1e-12)
    # b_g = +60: skips carry relative weight ~e^-60, so the result is sliding-window attention
    out40, lse40, _ = oracle.fwd(q, kk, v, np.zeros_like(w_g), np.full(2, 60.0, np.float32), k, 4, 9)
    np.testing.assert_allclose(out40, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse40, lse_ref, rtol=0, atol=1e-12)


def test_alpha_to_zero_is_skip_only():
    n, k, pi, S, d = 64, 4, 7, 8, 16
    q, kk, v, _, _ = _inputs(1, 2, n, d, seed=6)
    _, P = brute.masks(n, k, pi, S)
    rows = P.any(1)
    o_ref, lse_ref = _sdpa_masked(q, kk, v, np.where(rows[:, None], P, True))
    # b_g = -60: window keys carry relative weight ~e^-60
    out, lse, _ = oracle.fwd(q, kk, v, np.zeros((2, d), np.float32), np.full(2, -60.0, np.float32), k, pi, S)
    np.testing.assert_allclose(out[:, :, rows], o_ref[:, :, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[:, :, rows], lse_ref[:, :, rows], rtol=0, atol=1e-12)


def test_rows_sum_to_one_workload_shape():
    w = ps.WORKLOADS["bf16_n4k"]
    inp = ps.prefill_inputs(w)
    rows = np.random.default_rng(0).choice(w.B * w.H * w.n, 512, replace=False)
    _, _, rs = oracle.fwd_rows(inp["q"], inp["k"], inp["v"], inp["w_g"], inp["b_g"], w.k, w.pi, w.S, rows=rows)
    np.testing.assert_allclose(rs, 1.0, rtol=0, atol=1e-12)


def test_decode_equals_last_prefill_row():
    B, H, n, d, k, pi, S = 2, 3, 90, 16, 7, 11, 8
    q, kk, v, w_g, b_g = _inputs(B, H, n, d, seed=8)
    lengths = np.array([90, 53], dtype=np.int32)
    qd = np.stack([q[b, :, lengths[b] - 1] for b in range(B)])
    out, lse, _ = oracle.decode(qd, kk, v, w_g, b_g, k, pi, S, lengths=lengths)
    rows = np.array([(b * H + h) * n + lengths[b] - 1 for b in range(B) for h in range(H)])
    out_p, lse_p, _ = oracle.fwd_rows(q, kk, v, w_g, b_g, k, pi, S, rows=rows)
    np.testing.assert_array_equal(out, out_p)
    np.testing.assert_array_equal(lse, lse_p)


# ----------------------------------------------------------------------------------------------
# bidirectional variant: the window reaches k tokens both ways and the skips also reach i + m pi
# ----------------------------------------------------------------------------------------------

def _closed_form_totals_bidir(n, k, pi, S):
    # window: the token, min(i, k) before it, min(n - 1 - i, k) after it; skip m (m pi > k) lands
    # backward on n - m pi rows and forward on n - m pi rows
    sum_l = sum(1 + min(i, k) + min(n - 1 - i, k) for i in range(n))
    sum_p = sum(2 * max(0, n - m * pi) for m in range(1, S + 1) if m * pi > k)
    return sum_l, sum_p


@pytest.mark.parametrize("n,k,pi,S", [
    (256, 8, 16, 2), (4096, 128, 64, 4), (16, 3, 4, 5), (100, 12, 4, 9), (57, 0, 1, 60), (5, 9, 2, 3),
    (1, 0, 1, 1), (300, 64, 32, 2),
])
def test_bidir_index_totals_closed_form(n, k, pi, S):
    assert oracle.counts(n, k, pi, S, bidir=True) == _closed_form_totals_bidir(n, k, pi, S)


@pytest.mark.parametrize("n,k,pi,S", [
    (32, 3, 4, 5), (48, 5, 7, 9), (33, 0, 1, 40), (64, 16, 8, 4), (64, 16, 16, 3), (20, 6, 3, 10), (17, 4, 5, 0),
])
def test_bidir_index_sets_match_dense_masks(n, k, pi, S):
    W, P = brute.masks(n, k, pi, S, bidir=True)
    for i in range(n):
        L_o, P_o = oracle.index_set(i, k, pi, S, n=n, bidir=True)
        assert L_o.tolist() == np.nonzero(W[i])[0].tolist()
        assert sorted(P_o.tolist()) == np.nonzero(P[i])[0].tolist()
        assert not set(L_o.tolist()) & set(P_o.tolist())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n,k,pi,S,d", [(32, 3, 4, 5, 16), (48, 5, 7, 9, 8), (64, 16, 16, 3, 12), (7, 2, 9, 3, 16)])
def test_bidir_oracle_matches_dense_brute_force(dtype, n, k, pi, S, d):
    q, kk, v, w_g, b_g = _inputs(2, 3, n, d, seed=n * 37 + k, dtype=dtype)
    out, lse, rs = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S, bidir=True)
    out_b, lse_b, _ = brute.attention(q, kk, v, w_g, b_g, k, pi, S, bidir=True)
    np.testing.assert_allclose(out, out_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(rs, 1.0, rtol=0, atol=1e-12)


def test_bidir_oracle_matches_torch_sdpa():
    n, k, pi, S, d = 40, 6, 5, 7, 16
    q, kk, v, w_g, b_g = _inputs(1, 2, n, d, seed=17)
    _, _, bias = brute.attention(q, kk, v, w_g, b_g, k, pi, S, bidir=True)
    tq, tk, tv = (torch.from_numpy(brute.widen(x)) for x in (q, kk, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(bias))
    out, lse, _ = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S, bidir=True)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    scores = torch.einsum("bhid,bhjd->bhij", tq, tk) / math.sqrt(d) + torch.from_numpy(bias)
    np.testing.assert_allclose(lse, torch.logsumexp(scores, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_bidir_reversing_the_sequence_reverses_the_result():
    # the two-sided rule is symmetric under i -> n - 1 - i, so reversing q, k, v along the sequence
    # must reverse out and lse; a one-sided slip (a short forward window, a missing forward skip,
    # an off-by-one at the sequence end) breaks the symmetry
    n, k, pi, S, d = 61, 5, 7, 8, 16
    q, kk, v, w_g, b_g = _inputs(1, 2, n, d, seed=21)
    out, lse, _ = oracle.fwd(q, kk, v, w_g, b_g, k, pi, S, bidir=True)
    rev = lambda a: np.ascontiguousarray(a[:, :, ::-1])  # noqa: E731
    out_r, lse_r, _ = oracle.fwd(rev(q), rev(kk), rev(v), w_g, b_g, k, pi, S, bidir=True)
    np.testing.assert_allclose(out_r[:, :, ::-1], out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_r[:, :, ::-1], lse, rtol=0, atol=1e-12)


def test_bidir_alpha_to_one_is_two_sided_sliding_window():
    n, k, d = 64, 6, 16
    q, kk, v, w_g, _ = _inputs(1, 2, n, d, seed=23)
    pos = np.arange(n)
    two_sided = np.abs(pos[:, None] - pos[None, :]) <= k
    o_ref, lse_ref = _sdpa_masked(q, kk, v, two_sided)
    out, lse, _ = oracle.fwd(q, kk, v, np.zeros_like(w_g), np.full(2, 60.0, np.float32), k, 4, 9, bidir=True)
    np.testing.assert_allclose(out, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_bidir_last_row_equals_causal_last_row_without_forward_keys():
    # the last row has no key after it, so its two-sided sets are its causal sets
    n, k, pi, S, d = 50, 4, 6, 7, 8
    q, kk, v, w_g, b_g = _inputs(1, 2, n, d, seed=29)
    rows = np.array([n - 1, 2 * n - 1])
    o_b, l_b, _ = oracle.fwd_rows(q, kk, v, w_g, b_g, k, pi, S, rows=rows, bidir=True)
    o_c, l_c, _ = oracle.fwd_rows(q, kk, v, w_g, b_g, k, pi, S, rows=rows)
    np.testing.assert_array_equal(o_b, o_c)
    np.testing.assert_array_equal(l_b, l_c)
