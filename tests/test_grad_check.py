"""The backward parity check itself (tests/gpu_util.py grad_close), on the CPU: mistakes planted in a
copy of the oracle's gradients must fail it, and the roundings the tensor-core path makes on
purpose must pass it.  The shapes are the smoke test's and the bf16_n4k_bwd workload's first
sequence, where the gate gradients do not cancel."""
import math

import numpy as np
import pytest

import oracle
import pi_synth as ps
from tests.gpu_util import gate_scales, grad_close, no_skip_anywhere

NAMES = ("dq", "dk", "dv", "dw_g", "db_g")


def _ref(B, H, n, d, k, pi, S, seed):
    q = ps.normal((B, H, n, d), seed=seed, stream=1)
    kk = ps.normal((B, H, n, d), seed=seed, stream=2)
    v = ps.normal((B, H, n, d), seed=seed, stream=3)
    dO = ps.normal((B, H, n, d), seed=seed, stream=6)
    w_g = ps.normal((H, d), seed=seed, stream=4, std=1 / math.sqrt(d), dtype="f32")
    b_g = ps.normal((H,), seed=seed, stream=5, std=0.7, dtype="f32")
    *ref, terms = oracle.bwd(q, kk, v, w_g, b_g, ps.bf16_bits_to_f32(dO).astype(np.float64), k, pi, S,
                             return_terms=True)
    return ref, gate_scales(q, terms)


SHAPES = [(1, 2, 512, 64, 32, 16, 8, 3),     # the smoke test's backward
          (1, 1, 4096, 64, 128, 64, 4, 0)]   # one sequence of bf16_n4k_bwd


@pytest.fixture(scope="module", params=SHAPES, ids=["smoke", "n4k"])
def case(request):
    B, H, n, d, k, pi, S, seed = request.param
    assert not no_skip_anywhere(n, k, pi, S)
    return _ref(B, H, n, d, k, pi, S, seed)


def _close(name, g, r, scales):
    rss_dw, rss_db = scales
    return grad_close(name, g, r, "tc", rss_dw if name == "dw_g" else rss_db if name == "db_g" else None)


def test_exact_and_rounded_gradients_pass(case):
    ref, scales = case
    rng = np.random.default_rng(1)
    for name, r in zip(NAMES, ref):
        assert _close(name, r, r, scales)[0]
        # a relative perturbation of 2^-9 per element, random signs: a bf16 rounding
        noisy = r * (1 + rng.choice([-1.0, 1.0], size=r.shape) * 2.0 ** -9)
        ok, msg = _close(name, noisy, r, scales)
        assert ok, msg


@pytest.mark.parametrize("mutant", ["db_g zero", "dw_g half", "db_g sign", "dw_g transposed head", "dq zero row"])
def test_planted_mistakes_fail(case, mutant):
    ref, scales = case
    got = [np.array(r, copy=True) for r in ref]
    if mutant == "db_g zero":
        got[4][:] = 0.0
    elif mutant == "dw_g half":
        got[3] *= 0.5
    elif mutant == "db_g sign":
        got[4] = -got[4]
    elif mutant == "dw_g transposed head":
        got[3] = got[3][::-1].copy() if got[3].shape[0] > 1 else got[3][:, ::-1].copy()
    elif mutant == "dq zero row":
        got[0][0, 0, 7] = 0.0
        if not np.any(ref[0][0, 0, 7]):
            pytest.skip("row already zero")
    bad = [name for name, g, r in zip(NAMES, got, ref) if not _close(name, g, r, scales)[0]]
    assert bad, f"{mutant} passed the check"


def test_no_skip_anywhere():
    assert no_skip_anywhere(128, 16, 32, 0) and no_skip_anywhere(200, 300, 16, 20) and no_skip_anywhere(1, 0, 1, 1)
    assert not no_skip_anywhere(300, 20, 9, 5)


def test_zero_gate_gradients_get_a_noise_bound_not_a_free_pass():
    # S = 0: every row's dz cancels and the true gate gradients are zero; the bound is the rounding
    # of D_i summed over rows, far below a gate gradient of the size a problem with skips has
    (ref, scales) = _ref(1, 2, 256, 64, 16, 32, 0, 5)
    assert np.max(np.abs(ref[4])) < 1e-12
    rss_dw, rss_db = scales
    assert grad_close("db_g", ref[4] + 2 * 2.0 ** -9 * rss_db, ref[4], "tc", rss_db)[0]
    assert not grad_close("db_g", ref[4] + 4 * 2.0 ** -9 * rss_db, ref[4], "tc", rss_db)[0]

