"""The N > 1 plumbing of bench.py on the CPU: ranks are replicas (no collective on the
data path), and the only exchanges are the barrier and the max of the step time over
ranks. Two gloo ranks in spawned processes check the max and the barrier; the oracle
arm is run by rank 0 alone."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._dist = dist
        dist_max = bench.make_dist_max(device="cpu")
        bench.dist_barrier()
        got = [dist_max(t) for t in times[rank]]          # same collective steps, same order, every rank
        bench.dist_barrier()
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def _run_ranks(world, times):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_step_time_is_the_max_over_ranks():
    # rank 1 is slower on the first measurement, rank 0 on the second: every rank
    # reports the slower one each time
    res = _run_ranks(2, {0: [10.0, 7.5], 1: [12.25, 3.0]})
    assert res[0] == res[1] == [12.25, 7.5]


def test_single_process_needs_no_group():
    import bench
    assert bench._dist is None
    assert bench.make_dist_max(device="cpu")(4.5) == 4.5
    bench.dist_barrier()                                  # no group: a no-op


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(bench, "oracle_setup", lambda *a, **k: pytest.fail("rank 1 must not run the oracle"))
    assert bench.run_reference(bench.argparse.Namespace(steps=1, warmup=0)) is None
    assert capsys.readouterr().out == ""


def test_bench_started_as_one_process_spawns_its_ranks():
    # `bench.py --gpus 2` without torch.distributed.run around it starts the two ranks
    # itself (torch.distributed.run, one process per GPU); here the oracle arm, which
    # needs no GPU: rank 0 alone prints the line, rank 1 exits 0 without work
    import json
    import subprocess
    import bench
    cmd = bench.spawn_command(["--impl", "reference", "--gpus", "2"], 2, 29999)
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=2" in cmd
    assert "--master-addr=127.0.0.1" in cmd and cmd[-2:] == ["--gpus", "2"]
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env["OMP_NUM_THREADS"] = "2"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
