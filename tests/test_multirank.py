"""The multi-rank plumbing of bench.py, run as two gloo ranks on CPU: both
ranks see the slowest rank's time, the whole-job value counts the work of all
ranks over that time, every rank draws its own batch of the workload, and the
reference arm runs on rank 0 only. (The GPU path uses the same functions over
NCCL; the workload has no data-path collective.)"""
import hashlib
import json
import multiprocessing as mp
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import workloads as W
    group = bench.init_ranks("gloo", timeout_s=60)
    t_local = 1.0 + 0.5 * group.rank  # rank 1 is the slow one
    group.barrier()
    t_max = group.max(t_local)
    value = bench.weak_scaling_value(10.0, group.world, t_max)
    w = W.WORKLOADS["tiny_mha_s128_d64"]
    mine = W.Prefill(**{**w.__dict__, "seed": w.seed + bench.rank_seed_shift(group.rank)})
    q = W.make_prefill_inputs(mine)["q"]
    world_seen = group.world
    group.close()
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump({"world": world_seen, "t_max": t_max, "value": value,
                   "q_hash": hashlib.sha256(q.tobytes()).hexdigest()}, f)


def test_two_gloo_ranks_take_the_max_time_and_draw_their_own_batches(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert [p.exitcode for p in procs] == [0, 0]
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(2)]
    assert all(r["world"] == 2 for r in res)
    assert all(r["t_max"] == 1.5 for r in res)
    assert all(abs(r["value"] - 10.0 * 2 / 1.5) < 1e-12 for r in res)
    assert res[0]["q_hash"] != res[1]["q_hash"]


def test_world_size_one_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    group = bench.init_ranks("gloo")
    assert (group.world, group.rank) == (1, 0)
    group.barrier()
    assert group.max(3.25) == 3.25
    group.close()


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    import bench

    class Args:
        steps, warmup, gpus = 1, 3, 2

    assert bench.reference_arm(Args) == 0
    assert capsys.readouterr().out == ""


def test_launch_plan_follows_gpus_and_world_size():
    import bench
    assert bench.launch_plan(1, {}) == "single"
    assert bench.launch_plan(2, {}) == "spawn"
    assert bench.launch_plan(4, {"WORLD_SIZE": "4"}) == "rank"
    assert bench.launch_plan(1, {"WORLD_SIZE": "1"}) == "single"
    with pytest.raises(SystemExit):
        bench.launch_plan(8, {"WORLD_SIZE": "2"})


def test_bench_gpus_two_launches_two_ranks_with_their_own_batches():
    """`bench.py --gpus 2` without torchrun relaunches itself as two ranks;
    the CPU rehearsal (gloo) shows world 2, two different input batches and
    the slowest rank's time."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--plumbing-check"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["gpus_flag"] == 2
    assert len(line["rank_input_digests"]) == 2 and len(set(line["rank_input_digests"])) == 2
    assert line["t_max"] == 1.25 and abs(line["value"] - 2 / 1.25) < 1e-12
