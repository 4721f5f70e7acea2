"""Host-side logic of bench.py (CPU only): algorithmic work counts, traffic lookup, and the
multi-rank timing reduction under a 2-rank gloo process group."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

import bench
import oracle
import pi_synth as ps

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_index_totals_agree_with_oracle_enumeration():
    for name in ("tiny_f32", "bf16_n4k", "bf16_n32k", "bf16_n128k"):
        w = ps.WORKLOADS[name]
        assert bench.index_totals(w.n, w.k, w.pi, w.S) == oracle.counts(w.n, w.k, w.pi, w.S)


def test_index_totals_bidirectional_agree_with_oracle_enumeration():
    for n, k, pi, S in [(4096, 128, 64, 4), (300, 400, 16, 40), (1, 0, 1, 1), (777, 0, 1, 70), (2000, 100, 300, 9)]:
        assert bench.index_totals(n, k, pi, S, bidir=True) == oracle.counts(n, k, pi, S, bidir=True)


def test_work_of_the_default_workload():
    w = ps.WORKLOADS["bf16_n4k"]
    tokens, flops, bytes_ = bench.work(w)
    assert tokens == 4096
    # 8 heads x (520128 window + 7744 skip) pairs x 4 d flops, plus the gate
    assert flops == 8 * (4 * 64 * (520128 + 7744) + 2 * 64 * 4096)
    assert bytes_ == 8 * (4 * 4096 * 64 * 2 + 4 * 4096)


def test_decode_work():
    w = ps.WORKLOADS["decode_bf16"]
    tokens, flops, bytes_ = bench.work(w)
    assert tokens == 64
    assert bytes_ == 64 * 32 * (2 * 1056 * 128 * 2 + 2 * 128 * 2 + 4)


def test_traffic_line_needs_the_current_source(tmp_path, monkeypatch):
    files = bench.KERNEL_FILES["prefill"]
    sha = bench.source_hash(files)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({"records": [
        {"workload": "bf16_n4k", "bytes_per_step": 123, "files": files, "source_sha": sha, "path": "auto"},
        {"workload": "bf16_n4k", "bytes_per_step": 77, "files": files, "source_sha": sha, "path": "tc_fused"},
        {"workload": "bf16_n32k", "bytes_per_step": 9, "files": files, "source_sha": "stale"}]}))
    real_root = bench.ROOT
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "periodic_sparse_attention_b200")
    os.symlink(os.path.join(real_root, "periodic_sparse_attention_b200", "csrc"),
               tmp_path / "periodic_sparse_attention_b200" / "csrc")
    assert bench.profiled_traffic("bf16_n4k") == 123
    assert bench.profiled_traffic("bf16_n4k", "tc_fused") == 77
    assert bench.profiled_traffic("bf16_n4k", "simt") is None  # a record of another path does not apply
    assert bench.profiled_traffic("bf16_n32k") is None
    assert bench.profiled_traffic("bf16_n128k") is None


def test_default_workload_is_the_largest_single_gpu_prefill():
    w = ps.WORKLOADS[bench.DEFAULT_WORKLOAD]
    prefills = [x for x in ps.WORKLOADS.values() if x.kind == "prefill"]
    assert w.kind == "prefill" and w.B * w.H * w.n == max(x.B * x.H * x.n for x in prefills)
    assert (w.B, w.H, w.n, w.d, w.k, w.pi, w.S) == (1, 32, 131072, 128, 512, 1024, 16)


def test_committed_traffic_records_are_well_formed():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)["records"]
    for r in recs:
        assert r["workload"] in ps.WORKLOADS and r["bytes_per_step"] > 0 and "path" in r
        assert os.path.exists(os.path.join(ROOT, "profiles", r["profile"]))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, _ = bench.dist_env()
    got = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    with open(os.path.join(out_dir, f"r{r}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "max": got}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{i}.json")) for i in range(2)]
    assert [r["max"] for r in res] == [15.0, 15.0]
    assert [r["world"] for r in res] == [2, 2]


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_f32", "--cpu-budget", "0.3"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def _shard_rank_main(rank, world, port, out_dir):
    import dataclasses

    import numpy as np
    import torch
    import torch.distributed as dist

    from periodic_sparse_attention_b200 import shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # the bf16_n128k recipe's index rule on a short sequence: the halo spans several periods
    w = dataclasses.replace(ps.WORKLOADS["bf16_n128k"], name="n128k_short", H=2, n=6000, k=100, pi=64, S=16)
    plan = bench.shard_plan(w, world, rank)
    host = ps.prefill_rows(w, plan["s0"], plan["s1"], 0)
    k_loc = torch.from_numpy(host["k"].view(np.int16))
    v_loc = torch.from_numpy(host["v"].view(np.int16))
    k_ext, v_ext, kv0 = shard.exchange_halo(k_loc, v_loc, w.n, w.k, w.pi, w.S, align=w.pi)
    full = ps.prefill_inputs(w, 0)
    ok = (kv0 == plan["kv0"] and k_ext.shape[2] == plan["s1"] - kv0 and plan["halo_rows"] == plan["s0"] - kv0
          and np.array_equal(k_ext.numpy().view(np.uint16), full["k"][:, :, kv0:plan["s1"]])
          and np.array_equal(v_ext.numpy().view(np.uint16), full["v"][:, :, kv0:plan["s1"]]))
    with open(os.path.join(out_dir, f"s{rank}.json"), "w") as f:
        json.dump({"ok": bool(ok), "plan": {k: v for k, v in plan.items() if k in ("s0", "s1", "kv0", "halo_rows")}}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_shard_step_plan_and_halo_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_shard_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn")
    res = [json.load(open(tmp_path / f"s{i}.json")) for i in range(2)]
    assert all(r["ok"] for r in res), res
    # blocks of whole periods (pi = 64): 47 and 46 periods, the second taking the 48 rows past the last
    assert res[0]["plan"] == {"s0": 0, "s1": 47 * 64, "kv0": 0, "halo_rows": 0}
    assert res[1]["plan"] == {"s0": 47 * 64, "s1": 6000, "kv0": 47 * 64 - 16 * 64, "halo_rows": 16 * 64}
