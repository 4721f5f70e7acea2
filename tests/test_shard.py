"""Sequence sharding on the host: the row blocks, the halo plan, and the halo exchange itself
between gloo ranks on the CPU (the same torch.distributed point-to-point calls run over NCCL on
GPUs).  The shard kernel is checked against the oracle in test_gpu_shard.py."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from periodic_sparse_attention_b200 import shard


@pytest.mark.parametrize("n,world", [(1, 1), (10, 3), (4096, 4), (7, 8), (1000, 7)])
def test_shard_bounds_tile_the_sequence(n, world):
    blocks = [shard.shard_bounds(n, world, r) for r in range(world)]
    assert blocks[0][0] == 0 and blocks[-1][1] == n
    for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in blocks]
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("n,world,align", [(131072, 3, 1024), (131072, 8, 1024), (6000, 4, 64), (100, 8, 16),
                                           (5000, 3, 2048)])
def test_aligned_shard_bounds_start_on_whole_units(n, world, align):
    blocks = [shard.shard_bounds(n, world, r, align) for r in range(world)]
    assert blocks[0][0] == 0 and blocks[-1][1] == n
    for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
        assert a1 == b0
    assert all(a % align == 0 for a, b in blocks)
    units = [(b - a) // align for a, b in blocks[:-1]] + [(blocks[-1][1] - blocks[-1][0]) // align]
    assert max(units) - min(units) <= 1  # whole units spread evenly; the last block adds the rest
    assert shard.shard_bounds(n, world, 0, 1) == shard.shard_bounds(n, world, 0)  # align 1: the plain split


@pytest.mark.parametrize("n,world,k,pi,S", [(131072, 3, 512, 1024, 16), (6000, 4, 100, 64, 16),
                                             (5000, 3, 300, 256, 1)])
def test_aligned_halo_plan_covers_the_rows_from_a_whole_period(n, world, k, pi, S):
    plan = shard.halo_plan(n, world, k, pi, S, align=pi)
    for dst in range(world):
        s0, s1 = shard.shard_bounds(n, world, dst, pi)
        kv0 = shard.halo_start(s0, s1, k, pi, S, pi)
        assert kv0 % pi == 0 and kv0 <= max(0, s0 - shard.reach(k, pi, S))
        rows = [r for src, d, g0, g1 in plan if d == dst for r in range(g0, g1)]
        assert rows == (list(range(kv0, s0)) if s1 > s0 else [])


def test_reach_counts_skips_only_outside_the_window():
    assert shard.reach(128, 64, 4) == 256        # skips m = 3, 4 exist: back to 4 * 64
    assert shard.reach(128, 64, 2) == 128        # m0 = 3 > S: no skip, the window only
    assert shard.reach(1024, 2048, 31) == 63488
    assert shard.reach(0, 1, 0) == 0


@pytest.mark.parametrize("n,world,k,pi,S", [(1000, 4, 40, 16, 30), (300, 3, 8, 16, 2), (4096, 4, 128, 64, 4),
                                             (100, 8, 0, 1, 0), (257, 5, 100, 7, 40), (5000, 2, 1024, 2048, 31)])
def test_halo_plan_covers_exactly_the_rows_each_shard_reads(n, world, k, pi, S):
    plan = shard.halo_plan(n, world, k, pi, S)
    w = shard.reach(k, pi, S)
    for dst in range(world):
        s0, s1 = shard.shard_bounds(n, world, dst)
        got = [(g0, g1) for src, d, g0, g1 in plan if d == dst]
        srcs = [src for src, d, _, _ in plan if d == dst]
        assert srcs == sorted(srcs) and all(src < dst for src in srcs)
        rows = [r for g0, g1 in got for r in range(g0, g1)]
        want = list(range(max(0, s0 - w), s0)) if s1 > s0 else []
        assert rows == want
        for src, d, g0, g1 in plan:
            if d == dst:
                a, b = shard.shard_bounds(n, world, src)
                assert a <= g0 < g1 <= b  # a rank sends only rows it owns


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _exchange_main(rank, world, port, n, k, pi, S, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    B, H, d = 2, 3, 8
    # the whole sequence, known to every rank here only to check the result
    full_k = torch.arange(B * H * n * d, dtype=torch.float32).reshape(B, H, n, d)
    full_v = -full_k
    s0, s1 = shard.shard_bounds(n, world, rank)
    k_ext, v_ext, kv0 = shard.exchange_halo(full_k[:, :, s0:s1].contiguous(), full_v[:, :, s0:s1].contiguous(), n,
                                            k, pi, S)
    ok = kv0 == max(0, s0 - shard.reach(k, pi, S)) and torch.equal(k_ext, full_k[:, :, kv0:s1]) and \
        torch.equal(v_ext, full_v[:, :, kv0:s1])
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(f"{int(ok)} {kv0} {k_ext.shape[2]}")
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,n,k,pi,S", [
    (2, 200, 8, 16, 3),        # halo within the previous rank
    (3, 300, 40, 16, 12),      # halo of 192 rows: reaches two ranks back
    (4, 100, 0, 1, 0),         # no halo at all
    (4, 130, 100, 7, 40),      # halo longer than the sequence before some ranks
])
def test_halo_exchange_between_gloo_ranks(tmp_path, world, n, k, pi, S):
    port = _free_port()
    mp.start_processes(_exchange_main, args=(world, port, n, k, pi, S, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    for r in range(world):
        ok, kv0, rows = open(tmp_path / f"r{r}.txt").read().split()
        s0, s1 = shard.shard_bounds(n, world, r)
        assert ok == "1", f"rank {r}: halo rows differ from the sequence's rows {kv0}..{s1}"
        assert int(rows) == s1 - int(kv0)
