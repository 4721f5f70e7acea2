"""Sequence sharding of the causal prefill across devices, one process per device.

Each rank owns a contiguous block of rows [s0, s1) of every (b, h) sequence.  Under the index
rule a row i reads keys back to i - max(k_win, S*pi) (skips only where m*pi > k_win), never
forward, so a rank needs the K/V rows [max(0, s0 - reach), s0) from the ranks before it and
nothing from the ranks after it.  The fixed strides make this exchange known in advance: one step
of point-to-point sends (NCCL over NVLink, or gloo on the host) before the compute, with no
collective over the whole group.  The compute is pi_attn_fwd_shard on the halo followed by the
rank's own rows.  (gist.science summaries of "pi-Attention: Periodic Sparse Transformers for
Efficient Long-Context Modeling": Dutch sections 2-3, English Hardware Efficiency.)

The host logic here (bounds, plan, exchange) holds no attention arithmetic; the kernels do all of
it.
"""
from __future__ import annotations

from . import pi_attn_fwd_shard


def shard_bounds(n: int, world: int, rank: int, align: int = 1) -> tuple[int, int]:
    """Rows [s0, s1) of a sequence of n rows owned by `rank` of `world`: contiguous blocks of whole
    units of `align` rows, the first ranks one unit longer, the last rank also taking the rows past
    the last whole unit.  With align = pi every block starts on a whole period, which lets a shard
    take the split path (pi_attn_fwd_shard)."""
    if world < 1 or not 0 <= rank < world or n < 0 or align < 1:
        raise ValueError(f"bad shard request n={n} world={world} rank={rank} align={align}")
    units, rest = divmod(n, align)
    base, extra = divmod(units, world)
    s0 = (rank * base + min(rank, extra)) * align
    s1 = s0 + (base + (1 if rank < extra else 0)) * align
    return s0, s1 + (rest if rank == world - 1 else 0)


def reach(k_win: int, pi: int, S: int) -> int:
    """How far back a row reads: the window's k_win, or the farthest skip S*pi when skips exist
    (m from k_win // pi + 1 to S)."""
    m0 = k_win // pi + 1
    return max(k_win, S * pi) if S >= m0 else k_win


def halo_start(s0: int, s1: int, k_win: int, pi: int, S: int, align: int = 1) -> int:
    """kv0, the first K/V row a shard [s0, s1) holds: s0 - reach, rounded down to a whole unit of
    `align` rows (so that, with align = pi, the halo too starts on a whole period), at least 0; s0
    for an empty shard."""
    if s1 <= s0:
        return s0
    lo = s0 - reach(k_win, pi, S)
    return max(0, (lo // align) * align)


def halo_plan(n: int, world: int, k_win: int, pi: int, S: int, align: int = 1) -> list[tuple[int, int, int, int]]:
    """The exchange step: (src, dst, g0, g1) for each rank dst and each earlier rank src whose
    rows intersect dst's halo [halo_start(...), s0): src sends rows [g0, g1) to dst.  Sorted by
    (dst, src), so for each dst the pieces come in row order."""
    plan = []
    for dst in range(world):
        s0, s1 = shard_bounds(n, world, dst, align)
        if s1 <= s0:
            continue
        lo = halo_start(s0, s1, k_win, pi, S, align)
        for src in range(dst):
            a, b = shard_bounds(n, world, src, align)
            g0, g1 = max(a, lo), min(b, s0)
            if g0 < g1:
                plan.append((src, dst, g0, g1))
    return plan


def exchange_halo(k_loc, v_loc, n: int, k_win: int, pi: int, S: int, group=None, align: int = 1):
    """One halo exchange.  k_loc, v_loc [B, H, s1 - s0, d] are this rank's rows; returns
    (k_ext, v_ext, kv0): the rows [kv0, s1) of the sequence, kv0 = halo_start(...).  Every rank of
    the group calls it with the same n, k_win, pi, S and align."""
    import torch
    import torch.distributed as dist

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    s0, s1 = shard_bounds(n, world, rank, align)
    if k_loc.shape[2] != s1 - s0 or v_loc.shape != k_loc.shape:
        raise ValueError(f"rank {rank}: k/v hold {k_loc.shape[2]} rows, the shard has {s1 - s0}")
    B, H, _, d = k_loc.shape
    peer = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    ops, pieces = [], []
    for src, dst, g0, g1 in halo_plan(n, world, k_win, pi, S, align):
        if dst == rank:
            kb = torch.empty((B, H, g1 - g0, d), dtype=k_loc.dtype, device=k_loc.device)
            vb = torch.empty_like(kb)
            ops += [dist.P2POp(dist.irecv, kb, peer(src), group), dist.P2POp(dist.irecv, vb, peer(src), group)]
            pieces.append((g0, kb, vb))
        if src == rank:
            ks = k_loc[:, :, g0 - s0:g1 - s0].contiguous()
            vs = v_loc[:, :, g0 - s0:g1 - s0].contiguous()
            ops += [dist.P2POp(dist.isend, ks, peer(dst), group), dist.P2POp(dist.isend, vs, peer(dst), group)]
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    kv0 = halo_start(s0, s1, k_win, pi, S, align)
    pieces.sort(key=lambda p: p[0])
    k_ext = torch.cat([p[1] for p in pieces] + [k_loc], dim=2)
    v_ext = torch.cat([p[2] for p in pieces] + [v_loc], dim=2)
    if k_ext.shape[2] != s1 - kv0:
        raise RuntimeError(f"rank {rank}: halo holds {k_ext.shape[2] - (s1 - s0)} rows, expected {s0 - kv0}")
    return k_ext, v_ext, kv0


def pi_attn_fwd_sharded(q_loc, k_loc, v_loc, w_g, b_g, n: int, k_win: int, pi: int, S: int, group=None,
                        stream=None, align: int = 1):
    """The causal prefill of this rank's rows [s0, s1) = shard_bounds(n, world, rank, align) of every
    sequence of n rows (q_loc, k_loc, v_loc [B, H, s1 - s0, d], bf16 on this rank's device): the
    halo exchange, then the shard kernel (align = pi lets every shard take the split path where
    the shape prefers it).  Returns (out, lse) for the rank's rows; empty shards return empty
    tensors."""
    import torch
    import torch.distributed as dist

    k_ext, v_ext, kv0 = exchange_halo(k_loc, v_loc, n, k_win, pi, S, group, align)
    s0, s1 = shard_bounds(n, dist.get_world_size(group), dist.get_rank(group), align)
    if s1 == s0:
        B, H, _, d = q_loc.shape
        return torch.empty_like(q_loc), torch.empty((B, H, 0), dtype=torch.float32, device=q_loc.device)
    return pi_attn_fwd_shard(q_loc, k_ext.contiguous(), v_ext.contiguous(), w_g, b_g, k_win, pi, S, s0, kv0,
                             stream=stream)
