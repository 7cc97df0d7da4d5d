"""The replicas path of bench.py on two CPU ranks (gloo): the slowest rank's time sets the
whole-job rate, and every rank takes the same collective steps."""
import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_seconds = [0.010, 0.025][rank]
    slowest = bench.max_over_ranks(local_seconds, world, dist, "cpu")
    rate = bench.whole_job_rate(16384, 10, world, slowest)
    dist.barrier()
    out[rank] = (slowest, rate)
    dist.destroy_process_group()


def test_two_rank_rate_uses_the_slowest_rank():
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    slowest, rate = res[0]
    assert slowest == pytest.approx(0.025)
    assert rate == pytest.approx(2 * 16384 * 10 / 0.025)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1) == 0.5
    assert bench.whole_job_rate(100, 4, 1, 2.0) == 200.0


def _bench(args, env_extra=None):
    import json
    import subprocess
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       env=env, timeout=300)
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    return r.returncode, lines, r.stderr


def test_gpus_flag_launches_one_rank_per_device_count():
    """bench.py --gpus 2 started as a plain process launches two ranks itself (torch.distributed.run),
    and rank 0 alone prints one line that counts both."""
    rc, lines, err = _bench(["--gpus", "2", "--stub", "--steps", "3", "--warmup", "1"])
    assert rc == 0, err[-2000:]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["value"] > 0


def test_gpus_flag_and_world_size_must_agree():
    rc, lines, err = _bench(["--gpus", "2", "--stub"], {"WORLD_SIZE": "3", "RANK": "0"})
    assert rc == 2 and not lines
    assert "WORLD_SIZE" in err


def test_single_gpu_runs_in_process():
    rc, lines, err = _bench(["--stub", "--steps", "2", "--warmup", "1"])
    assert rc == 0, err[-2000:]
    assert lines[0]["n_gpus"] == 1


def test_reference_arm_prints_on_rank_zero_only():
    """The reference arm under N ranks: rank 0 times the oracle and prints the one line (counting N
    GPUs); any other rank exits 0 at once without work or output."""
    rc, lines, err = _bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"])
    assert rc == 0, err[-2000:]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    rc, lines, err = _bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"],
                            {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert rc == 0 and not lines, err[-2000:]
