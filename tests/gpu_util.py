"""Helpers shared by the GPU parity tests: moving generator output to the device and back, and
the comparison metrics with the operator's tolerances."""
import math

import numpy as np
import torch

import pi_synth as ps

# Tolerances of the CUDA path against the fp64 oracle, on the same stored inputs.
#   fp32 storage: max-abs 1e-5 on out and on lse.
#   bf16 storage (fp32 accumulation): max-abs 2e-2 and relative L2 5e-3 on out; lse max-abs 1e-3
#   (fp32 logits and sums; the bf16 rounding of the probabilities fed to the P.V product does not
#   enter lse).
TOL = {
    "f32": dict(out_abs=1e-5, out_rel_l2=1e-5, lse_abs=1e-5),
    "bf16": dict(out_abs=2e-2, out_rel_l2=5e-3, lse_abs=1e-3),
}


def to_dev(a: np.ndarray, dtype: str, device="cuda"):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def from_dev(t) -> np.ndarray:
    """Device tensor -> float64 numpy (bf16 widened exactly)."""
    if t.dtype == torch.bfloat16:
        return ps.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.float().cpu().numpy().astype(np.float64)


def metrics(got_out, ref_out, got_lse=None, ref_lse=None):
    d = got_out - ref_out
    m = {
        "out_abs": float(np.max(np.abs(d))) if d.size else 0.0,
        "out_rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(ref_out), 1e-300)) if d.size else 0.0,
        "finite": bool(np.all(np.isfinite(got_out))),
    }
    if got_lse is not None:
        m["lse_abs"] = float(np.max(np.abs(got_lse - ref_lse))) if got_lse.size else 0.0
        m["finite"] = m["finite"] and bool(np.all(np.isfinite(got_lse)))
    return m


def assert_close(m: dict, dtype: str, what: str = ""):
    tol = TOL[dtype]
    assert m["finite"], f"{what}: non-finite output {m}"
    assert m["out_abs"] <= tol["out_abs"], f"{what}: out max-abs {m['out_abs']:.3g} > {tol['out_abs']} {m}"
    assert m["out_rel_l2"] <= tol["out_rel_l2"], f"{what}: out rel-L2 {m['out_rel_l2']:.3g} {m}"
    if "lse_abs" in m:
        assert m["lse_abs"] <= tol["lse_abs"], f"{what}: lse max-abs {m['lse_abs']:.3g} > {tol['lse_abs']} {m}"


# Backward tolerances.  dq, dk, dv: relative L2 error, and max-abs error as a fraction of the
# gradient's largest magnitude.
#   simt: fp32 arithmetic against fp64 on the same bits.
#   tc:   the tensor-core path rounds on purpose -- the forward's P to bf16 (so its out, and the
#         D = dO . out taken from the fp32 output rows, carry a relative error of order 2^-9 per
#         weight) and dS to bf16 for dQ += dS K (2^-9 per element); each gradient carries a few
#         such roundings: 1e-2 (about 5 * 2^-9) for both measures.
# dw_g and db_g are sums over every row of dz_i q_i and dz_i, and a row's dz_i carries roundings:
#   - of D_i = dO_i . out_i, which the tensor-core path takes from an output computed with P rounded
#     to bf16: D_i - sum_j p_j dO_i . v_j = sum_j (p~_j - p_j) dO_i . v_j, each |p~_j - p_j| within
#     2^-9 p_j with an independent sign, so its spread is 2^-9 sqrt(sum_j p_j^2 (dO_i . v_j)^2); dz_i
#     takes it times (1 - alpha_i - sum_P p_j), and when every key of the row carries one prior the
#     true dz_i is exactly zero while this rounding remains;
#   - of dz_i's own sum, of the order of the unit roundoff times |dz_i|.
# Summed over rows with independent signs, a gate gradient's error has a spread of the unit
# roundoff times the root-sum-square of the rows' scales, sqrt(sum_j p_j^2 (dO_i . v_j)^2 + dz_i^2)
# (times |q_ic| for dw_g[h, c]).  gate_tol is 3 unit roundoffs (about 5 standard deviations of a
# uniform rounding) for the tensor-core path; the simt path, fp32 throughout, is held to 2^-16.
# This one rule also covers the problems whose true gate gradients are zero (no row has a skip).
GRAD_TOL = {
    "simt": dict(rel_l2=1e-4, max_abs_frac=1e-3, gate_tol=2.0 ** -16),
    "tc": dict(rel_l2=1e-2, max_abs_frac=1e-2, gate_tol=3 * 2.0 ** -9),
}


def no_skip_anywhere(n: int, k: int, pi: int, S: int) -> bool:
    """True when no row of a length-n sequence has a skip key (causal or bidirectional rule): the
    first surviving skip m0 = k // pi + 1 is past S, or m0 * pi reaches past the sequence."""
    m0 = k // pi + 1
    return S < m0 or m0 * pi > n - 1


def gate_scales(q_bits: np.ndarray, terms: np.ndarray):
    """Root-sum-square scales of the gate gradients' rounding: (for dw_g [H, d], for db_g [H]).
    q_bits: q [B, H, n, d] as stored (bf16 bits or fp32); terms: oracle.bwd(..., return_terms=True)'s
    per-row (dz_i, D_i, sum_j p_j^2 (dO_i . v_j)^2) [B, H, n, 3]."""
    q = ps.bf16_bits_to_f32(q_bits).astype(np.float64) if q_bits.dtype == np.uint16 else q_bits.astype(np.float64)
    s2 = terms[..., 2] + terms[..., 0] ** 2                                # [B, H, n]
    rss_dw = np.sqrt(np.einsum("bhn,bhnc->hc", s2, q * q))
    rss_db = np.sqrt(s2.sum(axis=(0, 2)))
    return rss_dw, rss_db


def grad_close(name: str, got: np.ndarray, ref: np.ndarray, path: str, gate_rss=None):
    """(ok, message) for one gradient of the backward against the oracle's.  gate_rss: for dw_g and
    db_g, the matching array of gate_scales."""
    tol = GRAD_TOL[path]
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if not np.all(np.isfinite(got)):
        return False, f"{name} not finite"
    err = np.abs(got - ref)
    mab = float(np.max(err)) if got.size else 0.0
    if name in ("dw_g", "db_g"):
        bound = tol["gate_tol"] * np.asarray(gate_rss, dtype=np.float64)
        worst = float(np.max(err / np.maximum(bound, 1e-300))) if got.size else 0.0
        return worst <= 1.0, f"{name} max-abs {mab:.3g}, worst error / bound {worst:.3g} (gate_tol {tol['gate_tol']:.3g})"
    scale = max(float(np.max(np.abs(ref))) if ref.size else 0.0, 1e-30)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    ok = rel <= tol["rel_l2"] and mab <= tol["max_abs_frac"] * scale
    return ok, f"{name} rel-L2 {rel:.3g} (bound {tol['rel_l2']}), max-abs {mab:.3g} (bound {tol['max_abs_frac'] * scale:.3g})"


def sampled_rows(w, count: int, seed: int = 0) -> np.ndarray:
    """`count` flat query rows drawn without replacement, plus for every (b, h) the boundary rows
    i in {0, k-1, k, k+1, pi, m0*pi, S*pi - 1, S*pi, n-1} (m0 = first skip outside the window)."""
    rng = np.random.default_rng(seed)
    total = w.B * w.H * w.n
    pick = rng.choice(total, size=min(count, total), replace=False)
    m0 = w.k // w.pi + 1
    bound = [0, w.k - 1, w.k, w.k + 1, w.pi, m0 * w.pi, w.S * w.pi - 1, w.S * w.pi, w.n - 1]
    bound = sorted({i for i in bound if 0 <= i < w.n})
    bh = np.arange(w.B * w.H)
    extra = (bh[:, None] * w.n + np.array(bound)[None, :]).reshape(-1)
    return np.unique(np.concatenate([pick, extra]))


def rel(a, b):
    return abs(a - b) / max(abs(b), 1e-300)


def tokens(w):
    return w.B * w.n if w.kind == "prefill" else w.B


def isqrt(x):
    return int(math.isqrt(x))
