"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Ranks shard the work as independent batches (weak scaling): no collective
touches the data path; the only cross-rank traffic is the barrier and the
max-over-ranks of the timed region. The --impl reference arm runs on rank 0
only; other ranks exit 0 without work.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from delta_rule_linear_falcon_b200 import inputs as I
    D = bench.Dist("gloo")
    try:
        # each rank draws a different batch from its own seed
        seed = bench.rank_seed(1, D.rank)
        s = I.make_seq(I.RULE_1, 1, 2, 8, 16, 16, seed=seed)
        my_ms = 10.0 + 5.0 * rank
        D.barrier()
        mx = D.max(my_ms)
        val = bench.weak_scaling_value(1000, D.world, mx)
        q.put((rank, seed, float(s.q.sum()), mx, val))
    finally:
        D.close()


def test_two_rank_weak_scaling_reduction():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = {r[1] for r in res}
    sums = {r[2] for r in res}
    assert len(seeds) == world and len(sums) == world        # independent batches
    assert all(r[3] == 15.0 for r in res)                     # max over ranks
    assert all(abs(r[4] - 2 * 1000 / 15e-3) < 1e-6 for r in res)


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
