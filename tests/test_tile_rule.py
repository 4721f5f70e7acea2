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
    st = np.zeros(4, np.int64)
    harness.tile_rule_sets(n, k, pi, S, 0, width, c.ctypes.data, idx.ctypes.data, st.ctypes.data)
    rc, ridx = oracle.index_table(n, k, pi, S, width)
    assert st[1] == 0, "a key was both a window key and a skip key"
    assert st[2] == 0, "a chunk class does not describe its chunk"
    assert st[3] == 0, "tiles not visited in increasing order"
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
    st = np.zeros(4, np.int64)
    harness.tile_rule_sets(n, k, pi, S, 1, width, c.ctypes.data, idx.ctypes.data, st.ctypes.data)
    rc, ridx = oracle.index_table(n, k, pi, S, width, bidir=True)
    assert st[1] == 0, "a key was both a window key and a skip key"
    assert st[2] == 0, "a chunk class does not describe its chunk"
    assert st[3] == 0, "tiles not visited in increasing order"
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
