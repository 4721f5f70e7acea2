"""Do the oracle's pins catch plausible mistakes?  (CPU only)

Each case plants one mistake in a private copy of the oracle's C source, compiles it, swaps it in
for the real oracle library, and runs the pin tests of test_oracle_pins.py.  Every mutant must
fail at least one pin; the unmodified source must fail none.  The mistakes are the ones a
hand-written oracle plausibly makes: a dropped term, a wrong sign or index, a transposed operand.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_backward as bpins
import tests.test_oracle_pins as pins
from tests.conftest import read_golden

SRC = os.path.join(os.path.dirname(oracle.__file__), "pi_oracle.c")

MUTANTS = {
    "priors_swapped": ("s[t] = tau * dot + (t < nL ? lL : lP);", "s[t] = tau * dot + (t < nL ? lP : lL);"),
    "window_one_short": ("int64_t a = i - kwin;", "int64_t a = i - kwin + 1;"),
    "tie_counted_as_skip": ("if (off <= kwin) continue;", "if (off < kwin) continue;"),
    "scale_dropped": ("s[t] = tau * dot + (t < nL ? lL : lP);", "s[t] = dot + (t < nL ? lL : lP);"),
    "prior_scaled": ("s[t] = tau * dot + (t < nL ? lL : lP);", "s[t] = tau * (dot + (t < nL ? lL : lP));"),
    "gate_on_scaled_query": ("z += qd[c] * (double)pr->w_g[h * d + c];",
                             "z += qd[c] * (double)pr->w_g[h * d + c] / sqrt((double)d);"),
    "gate_bias_dropped": ("double z = (double)pr->b_g[h];", "double z = 0.0;"),
    "lse_base2": ("*lse = M + log(Z);", "*lse = M + log2(Z);"),
    "keys_from_values": ("dot += qd[c] * load_elem(pr->k,", "dot += qd[c] * load_elem(pr->v,"),
    "last_skip_dropped": ("for (int64_t m = 1; m <= S; ++m) {", "for (int64_t m = 1; m < S; ++m) {"),
    "unnormalised": ("double p = exp(s[t] - M) / Z;", "double p = exp(s[t] - M);"),
    # bidirectional variant
    "bidir_forward_window_short": ("b = i + kwin;", "b = i + kwin - 1;"),
    "bidir_forward_skips_missing": ("if (bidir && i + off <= n - 1) {", "if (0 && i + off <= n - 1) {"),
    "bidir_forward_skip_tied_to_backward": ("if (bidir && i + off <= n - 1) {",
                                            "if (bidir && j >= 0 && i + off <= n - 1) {"),
}


def _pin_calls():
    g = read_golden
    yield lambda: pins.test_page_worked_example_score_counts(g)
    yield lambda: pins.test_page_worked_example_reach(g)
    for args in [(256, 8, 16, 2), (4096, 128, 64, 4), (100, 12, 4, 9), (300, 64, 32, 2)]:
        yield lambda a=args: pins.test_index_totals_closed_form(*a)
    for args in [(48, 5, 7, 9), (64, 16, 8, 4), (64, 16, 16, 3)]:
        yield lambda a=args: pins.test_index_sets_match_dense_masks(*a)
    for args in [(32, 3, 4, 5, 16), (64, 16, 8, 4, 32), (64, 16, 16, 3, 12)]:
        yield lambda a=args: pins.test_oracle_matches_dense_brute_force("bf16", *a)
    yield lambda: pins.test_brute_force_matches_torch_sdpa(40, 6, 5, 7, 16)
    yield pins.test_gate_closed_form_zero_query
    yield pins.test_gate_closed_form_zero_keys
    yield pins.test_alpha_to_one_is_causal_sliding_window
    yield pins.test_alpha_to_zero_is_skip_only
    for args in [(256, 8, 16, 2), (100, 12, 4, 9)]:
        yield lambda a=args: pins.test_bidir_index_totals_closed_form(*a)
    yield lambda: pins.test_bidir_index_sets_match_dense_masks(48, 5, 7, 9)
    yield lambda: pins.test_bidir_oracle_matches_dense_brute_force("bf16", 32, 3, 4, 5, 16)
    yield pins.test_bidir_reversing_the_sequence_reverses_the_result
    yield pins.test_bidir_alpha_to_one_is_two_sided_sliding_window


def _failures(lib):
    saved = oracle._lib_handle
    oracle._lib_handle = lib
    failed = 0
    try:
        for call in _pin_calls():
            try:
                call()
            except AssertionError:
                failed += 1
    finally:
        oracle._lib_handle = saved
    return failed


def _compile(src_text, tmp_path, name):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", str(c), "-o", str(so), "-lm"])
    return oracle.bind(ctypes.CDLL(str(so)))


def test_unmodified_oracle_passes_every_pin(tmp_path):
    assert _failures(_compile(open(SRC).read(), tmp_path, "clean")) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    lib = _compile(src.replace(old, new, 1), tmp_path, name)
    assert _failures(lib) >= 1, f"no pin caught the planted mistake {name!r}"


# Mistakes planted in the backward (gradients through out); each must fail a backward pin.
BWD_MUTANTS = {
    "bwd_gate_term_dropped": ("dq[i * d + c] += dz * (double)pr->w_g[h * d + c];", "dq[i * d + c] += 0.0;"),
    "bwd_prior_derivatives_swapped": ("dz += t < nL ? (1.0 - alpha) * ds : -alpha * ds;",
                                      "dz += t < nL ? -alpha * ds : (1.0 - alpha) * ds;"),
    "bwd_tau_dropped_in_dk": ("dk[j * d + c] += tau * ds * qd[c];", "dk[j * d + c] += ds * qd[c];"),
    "bwd_dv_from_ds": ("dv[j * d + c] += p[t] * g[c];", "dv[j * d + c] += (p[t] * (dpt - Dsum)) * g[c];"),
    "bwd_D_dropped": ("const double ds = p[t] * (dpt - Dsum);", "const double ds = p[t] * dpt;"),
    "bwd_gate_bias_grad_dropped": ("*db += dz;", "*db += 0.0;"),
}


def _bwd_failures(lib):
    saved = oracle._lib_handle
    oracle._lib_handle = lib
    failed = 0
    calls = [lambda: bpins.test_backward_matches_torch_autograd(40, 5, 7, 4, 8, False),
             lambda: bpins.test_backward_matches_torch_autograd(20, 30, 3, 5, 8, True),
             lambda: bpins.test_backward_matches_finite_differences(12, 3, 4, 2, False)]
    try:
        for call in calls:
            try:
                call()
            except AssertionError:
                failed += 1
    finally:
        oracle._lib_handle = saved
    return failed


def test_unmodified_backward_passes_its_pins(tmp_path):
    assert _bwd_failures(_compile(open(SRC).read(), tmp_path, "clean_bwd")) == 0


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_planted_backward_mistake_is_caught(name, tmp_path):
    old, new = BWD_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    lib = _compile(src.replace(old, new, 1), tmp_path, name)
    assert _bwd_failures(lib) >= 1, f"no backward pin caught the planted mistake {name!r}"
