"""The N > 1 plumbing of bench.py on the CPU: two gloo ranks, no GPU.

Each rank runs its own independent batches (the BitLinear path needs no
exchange step), so the only collectives are the barrier and the max over
ranks of the timed region; the reference arm runs on rank 0 alone.
"""
import json
import os
import socket
import subprocess
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    # each rank reports a different time: every rank must see the slowest one
    got = bench.max_over_ranks(1.5 * (rank + 1), world, torch.device("cpu"))
    # throughput is whole-job: tokens of all ranks over the slowest rank's time
    tokens = 16 * world * 10
    q.put((rank, got, tokens / (got / 1e3)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r for r, _, _ in res) == [0, 1]
    assert all(abs(v - 3.0) < 1e-12 for _, v, _ in res)
    assert all(abs(tp - 320 / 3e-3) < 1e-6 for _, _, tp in res)


def _bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_runs_on_rank0_only():
    common = ("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0")
    r1 = _bench({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"}, *common)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _bench({"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "2"}, *common)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["warmup"] >= 3
