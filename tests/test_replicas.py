"""Host logic of the multi-GPU replica path, on the CPU: two `gloo` ranks agree
on the slowest rank's time and on the whole-job throughput, and their
replicas use distinct weight seeds."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_quantization_group_b200 import workloads as wl
from post_weight_quantization_group_b200.replicas import (aggregate_throughput, max_over_ranks,
                                                          replica_layer)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took 1.0 + r seconds; every rank moved 10 GB
        t = max_over_ranks(1.0 + rank, dist)
        v = aggregate_throughput(10_000_000_000, t, world)
        seeds = sorted(wl.llama3_8b_layer_seeds(replica_layer(l, rank))["q_proj"] for l in range(32))
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{t} {v} {' '.join(map(str, seeds))}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_time_and_throughput(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    rows = [open(tmp_path / f"r{r}.txt").read().split() for r in range(world)]
    for row in rows:
        assert float(row[0]) == 2.0                    # the slowest rank
        assert float(row[1]) == pytest.approx(1e10)    # 2 x 10 GB / 2 s
    s0, s1 = set(rows[0][2:]), set(rows[1][2:])
    assert len(s0) == 32 and not (s0 & s1)             # distinct weights per replica


def test_single_process_is_identity():
    assert max_over_ranks(3.25) == 3.25
    assert aggregate_throughput(100, 2.0, 1) == 50.0
    with pytest.raises(ValueError):
        aggregate_throughput(100, 0.0, 1)


def test_replica_layers_distinct_across_ranks():
    seen = set()
    for rank in range(8):
        for layer in range(80):
            seen.add(replica_layer(layer, rank))
    assert len(seen) == 8 * 80
    with pytest.raises(ValueError):
        replica_layer(1000, 0)
