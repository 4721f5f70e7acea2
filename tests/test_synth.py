"""The seeded input generator (CPU only)."""
import numpy as np
import pytest

import pi_synth as ps


def test_philox_known_answers(golden):
    import os
    from tests.conftest import GOLDEN
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        lines = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(lines) == 3
    for words in lines:
        vals = [int(w, 16) for w in words]
        got = ps.philox4x32_10(vals[0:4], vals[4:6])
        assert got.tolist() == vals[6:10]


def test_rows_regenerate_exactly():
    shp = (2, 3, 100, 24)
    for dtype in ("bf16", "f32"):
        full = ps.normal(shp, seed=9, stream=3, dtype=dtype, scale_every=7, scale_factor=4.0)
        pick = np.array([0, 5, 99, 100, 357, 599])
        got = ps.rows(shp, pick, seed=9, stream=3, dtype=dtype, scale_every=7, scale_factor=4.0)
        assert np.array_equal(got, full.reshape(-1, 24)[pick])


def test_deterministic_and_streams_differ():
    a = ps.normal((1000,), seed=0, stream=1, dtype="f32")
    b = ps.normal((1000,), seed=0, stream=1, dtype="f32")
    c = ps.normal((1000,), seed=0, stream=2, dtype="f32")
    d = ps.normal((1000,), seed=1, stream=1, dtype="f32")
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_moments_and_bf16_rounding():
    x = ps.normal((1 << 20,), seed=0, stream=7, std=2.0, mean=0.5, dtype="f32")
    assert abs(x.mean() - 0.5) < 0.01 and abs(x.std() - 2.0) < 0.01
    xb = ps.normal((1 << 20,), seed=0, stream=7, std=2.0, mean=0.5, dtype="bf16")
    assert np.array_equal(xb, ps.f32_to_bf16_bits(x))
    # bf16 keeps 8 significant bits: relative rounding error at most half an ulp, 2^-8
    w = ps.bf16_bits_to_f32(xb)
    nz = x != 0
    assert np.max(np.abs(w[nz] - x[nz]) / np.abs(x[nz])) <= 2.0 ** -8


def test_key_row_scaling_recipe():
    w = ps.WORKLOADS["bf16_n32k"]
    shp = (1, 1, 1024, 16)
    plain = ps.bf16_bits_to_f32(ps.normal(shp, seed=0, stream=2, dtype="bf16"))
    scaled = ps.bf16_bits_to_f32(ps.normal(shp, seed=0, stream=2, dtype="bf16", scale_every=w.k_scale_every,
                                           scale_factor=w.k_scale_factor))
    rows = np.arange(1024)
    hit = rows % 256 == 0
    assert np.array_equal(scaled[0, 0, hit], 4 * plain[0, 0, hit])  # x4 is exact in bf16
    assert np.array_equal(scaled[0, 0, ~hit], plain[0, 0, ~hit])


def test_decode_storage_plan_covers_window_and_skips():
    pos = ps.decode_positions(65536, 1024, 2048, 31)
    assert pos.size == 1025 + 31
    assert pos.max() == 65535 and pos.min() == 65535 - 31 * 2048


@pytest.mark.parametrize("s0,s1", [(0, 4096), (1000, 2300), (4000, 4096), (17, 18)])
def test_prefill_rows_are_slices_of_the_full_inputs(s0, s1):
    # the sequence-sharded bench generates only its own rows; they must be the same values
    import dataclasses
    w = dataclasses.replace(ps.WORKLOADS["bf16_n32k"], name="n32k_small", H=2, n=4096)
    full = ps.prefill_inputs(w, 3)
    part = ps.prefill_rows(w, s0, s1, 3)
    for name in ("q", "k", "v"):
        assert np.array_equal(full[name][:, :, s0:s1], part[name]), name
    assert np.array_equal(full["w_g"], part["w_g"]) and np.array_equal(full["b_g"], part["b_g"])
