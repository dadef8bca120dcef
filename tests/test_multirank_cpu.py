"""The multi-rank (N > 1) host path of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank quantizes its own layer (weak scaling, no collective on the data path); the
only collectives are the barrier and the max-over-ranks reduction of the timed region,
and the reported value is the units all ranks processed over that time.  The ranks run
in their own interpreters (torch.distributed.run), not inside the test process.
"""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_units(tmp_path):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2", "--standalone",
           "--local-addr", "127.0.0.1", os.path.join(ROOT, "tests", "multirank_worker.py")]
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", OMP_NUM_THREADS="1", MULTIRANK_OUT=str(tmp_path))
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=180, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    res = {}
    for rank in range(2):
        d = json.loads((tmp_path / f"rank{rank}.json").read_text())
        res[d["rank"]] = d
    assert set(res) == {0, 1}
    for d in res.values():
        assert d["world"] == 2
        assert d["job_ms"] == pytest.approx(15.0)                          # max over ranks, on every rank
        assert d["value"] == pytest.approx(2 * 4096 * 4096 * 3 / 15e-3)    # all ranks' units / job time
    assert res[0]["seed"] != res[1]["seed"]                                # independent layers per rank


def test_single_process_path_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5, None, None) == 7.5
    assert bench.job_throughput(1, 100.0, 4, 2.0) == pytest.approx(100.0 * 4 / 2e-3)


def _clean_env():
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT", "LOCAL_WORLD_SIZE")}
    env["OMP_NUM_THREADS"] = "1"
    return env


def test_gpus_n_without_torchrun_launches_n_ranks_itself():
    """bench.py --gpus 2 started as a plain process becomes two ranks (torch.distributed.run
    on 127.0.0.1); the launch check joins them in a gloo group, so rank 0 sees world 2."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--rank-probe"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=180, cwd=ROOT, env=_clean_env())
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert lines[0]["world"] == 2 and lines[0]["rank_sum"] == 1.0


def test_gpus_n_that_disagrees_with_the_launcher_fails():
    env = _clean_env()
    env.update(WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--rank-probe"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert r.returncode != 0


def test_relaunch_command_shape():
    sys.path.insert(0, ROOT)
    import bench

    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "3"], 4, 29511)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "29511" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
