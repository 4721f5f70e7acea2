"""The tensor-core kernel's index logic (tile walk, per-row tile masks, chunk classes), compiled
from its own header with g++ and replayed on the CPU, against the oracle's index sets."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("tile") / "tile_rule.so")
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", os.path.join(HERE, "tile_rule_harness.cpp"),
                           "-o", so])
    lib = ctypes.CDLL(so)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.tile_rule_sets.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp]
    return lib


CASES = [
    (256, 8, 16, 2), (4096, 128, 64, 4), (32768, 256, 256, 8), (4000, 512, 1024, 16), (1000, 100, 37, 12),
    (333, 400, 16, 40), (200, 64, 32, 0), (300, 8, 1, 50), (513, 128, 64, 6), (130, 5, 7, 3), (640, 0, 128, 4),
    (385, 127, 129, 2), (1, 0, 1, 1), (2048, 1024, 2048, 31), (5000, 200, 300, 15), (777, 0, 1, 70),
    (1100, 256, 256, 8), (700, 64, 96, 6), (2049, 63, 65, 40), (1500, 300, 1, 3),
]


@pytest.mark.parametrize("n,k,pi,S", CASES)
def test_kernel_index_logic_matches_oracle(harness, n, k, pi, S):
    width = k + 1 + S
    c = np.zeros((n, 2), np.int32)
    idx = np.zeros((n, width), np.int32)
    st = np.zeros(6, np.int64)
    harness.tile_rule_sets(n, k, pi, S, 0, width, c.ctypes.data, idx.ctypes.data, st.ctypes.data)
    rc, ridx = oracle.index_table(n, k, pi, S, width)
    assert st[1] == 0, "a key was both a window key and a skip key"
    assert st[2] == 0, "a chunk class does not describe its chunk"
    assert st[3] == 0, "tiles not visited in increasing order"
    assert st[4] == 0, "the incremental tile cursor departs from the tile walk"
    assert st[5] == 0, "the incremental row skips depart from the row's tile mask"
    assert np.array_equal(c, rc)
    assert np.array_equal(idx, ridx)


BIDIR_CASES = [
    (256, 8, 16, 2), (4096, 128, 64, 4), (1000, 100, 37, 12), (333, 400, 16, 40), (200, 64, 32, 0), (300, 8, 1, 50),
    (513, 128, 64, 6), (130, 5, 7, 3), (640, 0, 128, 4), (385, 127, 129, 2), (1, 0, 1, 1), (2048, 100, 2048, 31),
    (5000, 200, 300, 15), (777, 0, 1, 70), (2049, 63, 65, 40), (1500, 300, 1, 3), (190, 1, 130, 2),
]


@pytest.mark.parametrize("n,k,pi,S", BIDIR_CASES)
def test_kernel_index_logic_matches_oracle_bidirectional(harness, n, k, pi, S):
    width = 2 * k + 1 + 2 * S
    c = np.zeros((n, 2), np.int32)
    idx = np.zeros((n, width), np.int32)
    st = np.zeros(6, np.int64)
    harness.tile_rule_sets(n, k, pi, S, 1, width, c.ctypes.data, idx.ctypes.data, st.ctypes.data)
    rc, ridx = oracle.index_table(n, k, pi, S, width, bidir=True)
    assert st[1] == 0, "a key was both a window key and a skip key"
    assert st[2] == 0, "a chunk class does not describe its chunk"
    assert st[3] == 0, "tiles not visited in increasing order"
    assert st[4] == 0, "the incremental tile cursor departs from the tile walk"
    assert st[5] == 0, "the incremental row skips depart from the row's tile mask"
    assert np.array_equal(c, rc)
    for i in range(n):
        nl, npk = rc[i]
        assert np.array_equal(idx[i, :nl], ridx[i, :nl])  # window keys, ascending
        assert sorted(idx[i, nl:nl + npk].tolist()) == sorted(ridx[i, nl:nl + npk].tolist())


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("n,k,pi,S", [(256, 8, 16, 2), (4096, 128, 64, 4), (1000, 100, 37, 12), (333, 400, 16, 40),
                                      (200, 64, 32, 0), (300, 8, 1, 50), (2049, 63, 65, 40), (640, 0, 128, 4),
                                      (1, 0, 1, 1), (1500, 300, 1, 3)])
def test_reader_walk_visits_exactly_the_reading_row_tiles(harness, n, k, pi, S, bidir):
    harness.reader_walk_tiles.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p, ctypes.c_void_p]
    nb = (n + 63) // 64
    maxper = nb
    tiles = np.full((nb, maxper), -1, np.int32)
    counts = np.zeros(nb, np.int32)
    assert harness.reader_walk_tiles(n, k, pi, S, int(bidir), maxper, tiles.ctypes.data, counts.ctypes.data) == 0
    cnt, idx = oracle.index_table(n, k, pi, S, bidir=bidir)
    expect = [set() for _ in range(nb)]
    for i in range(n):
        for j in idx[i, : cnt[i].sum()]:
            expect[j // 64].add(i // 64)
    for b in range(nb):
        assert set(tiles[b, : counts[b]].tolist()) == expect[b], (b, sorted(expect[b]), tiles[b, : counts[b]].tolist())


def test_residue_view_walks_give_exactly_the_needed_tiles(harness):
    # the split path's query walk (the dq and residue forward passes) and reader walk (the dk/dv
    # skip pass) over one residue class, against brute force: T rows a class, blocks of 128
    harness.residue_walk_mismatches.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    for T, S, m0 in [(1, 1, 1), (4, 3, 1), (64, 30, 3), (128, 8, 2), (256, 40, 9), (3000, 90, 11), (200, 5, 6),
                     (129, 200, 1), (700, 64, 64)]:
        assert harness.residue_walk_mismatches(T, S, m0, 128) == 0, (T, S, m0)
    rng = np.random.default_rng(11)
    for _ in range(300):
        T = int(rng.integers(1, 1500))
        m0 = int(rng.integers(1, 12))
        S = int(rng.integers(0, 150))
        assert harness.residue_walk_mismatches(T, S, m0, 128) == 0, (T, S, m0)


def test_bidirectional_residue_walk_covers_both_bands(harness):
    # the bidirectional split's residue pass: every tile holding a key of some row's backward or
    # forward band is walked once, and nothing outside the block's reach
    harness.residue_walk_bidir_errors.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    for T, S, m0 in [(1, 1, 1), (4, 3, 1), (64, 30, 3), (128, 8, 2), (256, 40, 9), (300, 90, 11), (200, 5, 6),
                     (129, 200, 1), (700, 64, 64)]:
        assert harness.residue_walk_bidir_errors(T, S, m0, 128) == 0, (T, S, m0)
    rng = np.random.default_rng(12)
    for _ in range(200):
        T = int(rng.integers(1, 1500))
        m0 = int(rng.integers(1, 12))
        S = int(rng.integers(0, 150))
        assert harness.residue_walk_bidir_errors(T, S, m0, 128) == 0, (T, S, m0)


def test_cursor_matches_walk_on_walks_built_by_field(harness):
    # band-only walks as the residue-class pass builds them (rows t of a residue view read keys
    # t - S .. t - m0: last is shifted down by m0 and may fall below i0 or below zero), and
    # random skip walks
    harness.cursor_vs_walk.argtypes = [ctypes.c_longlong] * 5 + [ctypes.c_int] * 4
    rng = np.random.default_rng(5)
    for _ in range(3000):
        T = int(rng.integers(1, 3000))
        q0 = int(rng.integers(0, (T + 127) // 128)) * 128
        Sr = int(rng.integers(0, 60))
        m0 = int(rng.integers(1, 8))
        last = min(q0 + 127, T - 1) - m0
        assert harness.cursor_vs_walk(q0, last, max(q0 - Sr, 0), last, T, 1, 0, 1, 0) == 0
        n = int(rng.integers(1, 5000))
        i0 = int(rng.integers(0, (n + 127) // 128)) * 128
        k = int(rng.integers(0, 700))
        pi = int(rng.integers(1, 400))
        S = int(rng.integers(0, 40))
        bidir = int(rng.integers(0, 2))
        lastr = min(i0 + 127, n - 1)
        hi = min(lastr + k, n - 1) if bidir else lastr
        assert harness.cursor_vs_walk(i0, lastr, max(i0 - k, 0), hi, n, pi, S, k // pi + 1, bidir) == 0


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("n,k,pi,S", [(256, 8, 16, 2), (700, 100, 37, 12), (333, 400, 16, 40), (200, 64, 32, 0),
                                      (300, 8, 1, 50), (513, 128, 64, 6), (130, 5, 7, 3), (640, 0, 128, 4),
                                      (385, 127, 129, 2), (1000, 40, 16, 30)])
def test_key_side_walk_gives_exactly_the_reading_rows(harness, n, k, pi, S, bidir):
    # the dk/dv pass's view: key blocks of 128 keys, 64-row reading tiles, per key its window rows
    # (a range) and its skip rows (KeyReaders), against the oracle's index sets transposed
    harness.key_side_mismatches.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p]
    width = (2 * k + 1 + 2 * S) if bidir else (k + 1 + S)
    c, idx = oracle.index_table(n, k, pi, S, width, bidir=bidir)
    reads = np.zeros((n, n), np.int8)
    for i in range(n):
        nl, npk = c[i]
        reads[i, idx[i, :nl]] = 1
        reads[i, idx[i, nl:nl + npk]] = 2
    assert harness.key_side_mismatches(n, k, pi, S, int(bidir), 128, reads.ctypes.data) == 0
