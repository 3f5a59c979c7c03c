"""The benchmark's multi-rank host logic on CPU: two gloo ranks, each an
independent replica, report the slowest rank's time and the whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [12.5, 20.0][rank]
    ms = bench.max_over_ranks(local_ms, world, device="cpu")
    rate = bench.job_rate(100, world, ms)
    out[rank] = (ms, rate)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, rate = res[rank]
        assert ms == 20.0
        assert rate == pytest.approx(2 * 100 / 0.020)


def test_single_rank_is_local():
    import bench
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.job_rate(10, 1, 5.0) == pytest.approx(2000.0)


@pytest.mark.parametrize("workload", ["tiny", "30b-sign", "30b-e16"])
def test_reference_arm_json_line(workload):
    """`bench.py --impl reference` runs the oracle on the host and prints one
    JSON line with the contract's keys, its cpu_baseline and e2e equal to the
    line's own value."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", workload, "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("moe-")
