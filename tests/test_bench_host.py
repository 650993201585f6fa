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
    rec = tmp_path / "rec.md"
    rec.write_text(f"kernel_sources_sha256_16: {bench.kernel_source_digest()}\n"
                   "traffic_bytes_per_launch_f32: 12345\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(rec))
    assert bench.recorded_traffic("f32") == 12345
    assert bench.recorded_traffic("bf16") is None
    rec.write_text("kernel_sources_sha256_16: 0000000000000000\ntraffic_bytes_per_launch_f32: 1\n")
    assert bench.recorded_traffic("f32") is None
