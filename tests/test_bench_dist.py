"""CPU coverage of the benchmark's multi-rank path (gloo, world size 2).

The scan shards over sequences with no exchange step, so the only cross-rank
logic is the timing reduction (max over ranks) and the weak-scaling throughput;
the reference arm must print from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms, k = bench.max_over_ranks([10.0 + 5 * rank, 1.0 + rank], world, "cpu")
    value = bench.weak_scaling_value(15, 100, ms, world)
    out[rank] = (ms, k, value)
    dist.barrier()
    dist.destroy_process_group()


def test_timing_is_the_max_over_ranks_and_throughput_scales_with_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    ms, k, value = res[0]
    assert ms == 15.0 and k == 2.0
    assert value == pytest.approx(2 * 15 * 100 / 0.015)


def test_reference_arm_prints_from_rank_zero_only():
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2")
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                            "tiny", "--steps", "1", "--warmup", "3", "--gpus", "2"],
                           capture_output=True, text=True, env=env, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    line = json.loads(outs[0])
    assert line["impl"] == "reference" and line["unit"] == "nodes/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert outs[1] == ""
