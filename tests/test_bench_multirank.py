"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Checks the max-over-ranks timing reduction, the weak-scaling accounting (all
ranks' bytes over the slowest rank's time), and that the reference arm runs on
rank 0 only (over every host core) while the other rank returns without work.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from nvfp4_microscaling_quantization_b200 import workloads as W
    bench.init_dist(world, "gloo")
    got_max = bench.max_over_ranks(1.5 + rank, world)
    bench.barrier(world)
    args = bench.parse_args(["--impl", "reference", "--steps", "2", "--warmup", "1"])
    line = bench.run_reference(args, world, rank, wl=W.small(), fraction=0.25)
    bench.barrier(world)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": got_max, "line": line}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["max"] == r1["max"] == 2.5
    assert r1["line"] is None                     # rank 1 did no work
    line = json.loads(r0["line"])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    from oracle.pool import host_cores
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == host_cores()
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_weak_scaling_value():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 3 steps x 1e9 bytes in 1.5 s (slowest rank) = 4 GB/s
    assert bench.weak_scaling_value(1e9, 3, 2, 1.5) == pytest.approx(4.0)
