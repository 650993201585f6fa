"""Host-side logic of bench.py, on the CPU: the multi-rank aggregation (max of
the per-rank device times, sum of the work) over a two-rank gloo group, the
per-rank seeds of the weak-scaling replicas, and the algorithmic byte counts
of the BEVFormer-base SCA workload."""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from scale_deformable_attention_03_b200 import inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, result_q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = [12.5, 30.25][rank]
    local_samples = [1000, 3000][rank]
    t, n = bench.aggregate(local_ms, local_samples, world)
    result_q.put((rank, t, n))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, t, n in got:
        assert t == 30.25      # the slowest rank's device time
        assert n == 4000       # all ranks' sampled points


def test_single_rank_aggregate_is_identity():
    assert bench.aggregate(7.0, 11, 1) == (7.0, 11)


def test_replica_seeds_are_distinct():
    seeds = [bench.rank_seed(r) for r in range(8)]
    assert seeds[0] == 1003 and len(set(seeds)) == 8


def test_algorithmic_bytes_bevformer_base():
    w = inputs.workload3()
    rows = int(w.bev_mask.any(-1).sum())
    hit_q = int(w.bev_mask.any(-1).any(0).sum())
    b = bench.algorithmic_bytes(w, rows, hit_q, 4)
    # value 189.4 MB, offsets 81.9, logits 41.0, rho 7.7, mask 0.96, out 41.0
    assert abs(b["step"] / 1e6 - 361.9) < 0.5
    assert 59000 < rows < 61000 and hit_q == w.Nq
    b16 = bench.algorithmic_bytes(w, rows, hit_q, 2)
    assert abs((b["step"] - b16["step"]) / 1e6 - 94.7) < 0.1


def test_config_is_json():
    args = bench.parse_args(["--gpus", "2"])
    json.dumps(bench.workload_config(args))
    assert args.steps >= 1 and args.warmup >= 3


def test_traffic_record_requires_matching_sources(tmp_path, monkeypatch):
    rec = tmp_path / "traffic.json"
    rec.write_text(json.dumps({"kernel_sources_sha256_16": bench.kernel_source_digest(),
                               "dram_bytes_per_launch": {"f32": 12345}}))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(rec))
    assert bench.recorded_traffic("f32") == 12345
    assert bench.recorded_traffic("bf16") is None
    rec.write_text(json.dumps({"kernel_sources_sha256_16": "0000000000000000",
                               "dram_bytes_per_launch": {"f32": 1}}))
    assert bench.recorded_traffic("f32") is None


class _FakeW:
    """The few workload fields the JSON line reads."""
    H, L, P = 8, 4, 8


def _stub_replica(args, rank, world, barrier):
    """Stands in for the device section: per-rank step times and work that
    depend on the rank's replica seed, with the section's barriers."""
    seed = bench.rank_seed(rank)
    barrier()   # before the timed steps
    barrier()   # after them
    barrier()   # before the end-to-end leg
    k = 1 + rank
    return {"w": _FakeW(), "bf16": False, "step_ms": [0.5 * k] * args.steps,
            "staged_ms": [0.51 * k] * args.steps, "gather_ms": [0.4 * k] * args.steps, "compact_ms": [0.05] * args.steps,
            "avg_ms": [0.05] * args.steps, "warm_gather_ms": 0.3,
            "samples_per_step": 1000 * k + seed % 7, "rows": 10, "seed": seed,
            "nbytes": {"step": 4_000_000, "gather": 5_000_000},
            "e2e_ms": 2.0 * k * args.e2e_steps, "h2d": 123, "d2h": 45, "clocks": None,
            "launches_per_step": 5}


def _bench_worker(rank, world, port, out_dir):
    import contextlib
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    args = bench.parse_args(["--gpus", str(world), "--steps", "4", "--warmup", "3",
                             "--e2e-steps", "2", "--cpu-seconds", "0", "--rows-iters", "0"])
    with open(os.path.join(out_dir, f"rank{rank}.out"), "w") as f, contextlib.redirect_stdout(f):
        rc = bench.run_native(args, backend="gloo", replica=_stub_replica)
    assert rc == 0


def test_bench_replica_path_two_ranks_gloo(tmp_path):
    """bench.run_native with two gloo ranks and a stubbed device section: the
    ranks' replicas get distinct seeds, rank 0 alone prints the line, and its
    value is all ranks' work over the slowest rank's time."""
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_bench_worker, args=(r, 2, port, str(tmp_path)))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert (tmp_path / "rank1.out").read_text() == ""
    line = json.loads((tmp_path / "rank0.out").read_text())
    s0, s1 = bench.rank_seed(0), bench.rank_seed(1)
    assert s0 != s1
    work = 4 * ((1000 + s0 % 7) + (2000 + s1 % 7))
    slowest_ms = 4 * 0.5 * 2
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert abs(line["value"] - work / (slowest_ms * 1e-3) / 1e9) < 1e-12
    assert abs(line["ms_per_step"] - slowest_ms / 4) < 1e-12
    e2e_work = 2 * ((1000 + s0 % 7) + (2000 + s1 % 7))
    assert abs(line["e2e"]["value"] - e2e_work / (2.0 * 2 * 2 * 1e-3) / 1e9) < 1e-12
    # rank 0's own stage times: the one-call step and the instrumented pass
    ms = line["step"]["ms"]
    assert abs(ms["step"] - 0.5) < 1e-12 and abs(ms["staged_step"] - 0.51) < 1e-12
    assert abs(ms["gather"] - 0.4) < 1e-12 and "sca_forward call" in line["step"]["timing"]
    assert line["gpu_launches"] == 5 * 4 and line["roofline"]["launch_ms"] == ms["gather"]
    assert "cpu_baseline" not in line and "next_rows" not in line
