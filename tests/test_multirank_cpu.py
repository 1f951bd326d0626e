"""The N > 1 host logic of bench.py on CPU: world-size-2 gloo ranks.

Each rank of a multi-GPU run processes its own full workload (weak scaling, no
collective on the data path); the only cross-rank steps are the barrier and the max
of the per-rank times.  These tests run that logic with the gloo backend.
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


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + rank * 5.0)      # per-rank step time (ms)
        q.put((rank, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_aggregate_is_whole_job_throughput():
    import bench
    b = bench.row_bytes()
    step = float(sum(b.values()))
    # two ranks, the slower one takes 10 ms per step: 2 * bytes / 10 ms
    assert bench.aggregate(step, 2, 10.0, 5) == pytest.approx(2 * step / 0.010 / 1e9)
    assert bench.aggregate(step, 1, 10.0, 1) == pytest.approx(step / 0.010 / 1e9)


def test_row_bytes_match_the_workload():
    import bench
    b = bench.row_bytes()
    rows = 32 * 2 * 8 * 32 * 4096
    assert b["quantize_cache"] == rows * (2 * 128 + 128 + 4)
    assert b["dequantize_cache"] == rows * (128 + 4 + 2 * 128)
    keys = 4 * 8 * 131072
    assert b["decode_qjl"] == keys * (32 + 2 + 128 + 4) + 256 * 128 * 2 + 4 * 32 * 128 * 6
    # quantize, 32 x (INT8 decode + combine), dequantize, QJL encode, value quantize,
    # tensor-core QJL decode + combine
    assert bench.LAUNCHES_PER_STEP == 1 + 32 * 2 + 3 + 2


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-scale", "0.25"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
