"""bench.py's multi-rank launcher, on the CPU: ``--gpus N`` outside a launcher starts N ranks
itself (torchrun, 127.0.0.1), every rank joins the process group, and rank 0 alone prints one
JSON line whose n_gpus is the world size. The ranks run the gloo self-test step instead of the
GPU step, so no device is needed."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _env():
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def test_relaunch_command_uses_loopback_and_same_args():
    cmd = bench.relaunch_command(4, ["--gpus", "4", "--steps", "7"])
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-3:] == ["--gpus", "4", "--steps", "7"][-3:]
    assert cmd[-5].endswith("bench.py")


def test_gpus_two_starts_two_ranks():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--launcher-selftest"], cwd=ROOT, env=_env(), capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout           # rank 0 alone prints
    j = json.loads(lines[0])
    assert j["n_gpus"] == 2 and j["sum_ranks"] == 3.0 and abs(j["max_time"] - 0.002) < 1e-12


def test_single_rank_selftest_runs_in_process():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--launcher-selftest"],
                       cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    j = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert j["n_gpus"] == 1 and j["sum_ranks"] == 1.0


def test_median_and_update_bytes():
    assert bench._median([3.0, 1.0, 2.0]) == 2.0
    assert bench._median([4.0, 1.0, 2.0, 3.0]) == 2.5
    # the algorithmic bytes of the headline update: X once + 4 passes over int32 ids
    assert bench.UPDATE_BYTES == 32 * 65536 * 128 * 2 + 4 * 32 * 65536 * 4


def _agree_rank(rank, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        # the ranks' own block counts differ; every rank must run the larger one
        out[rank] = bench._agree_max(3 + 2 * rank, dist)
    finally:
        dist.destroy_process_group()


def test_ranks_agree_on_the_number_of_timed_blocks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = bench._free_port()
        ps = [ctx.Process(target=_agree_rank, args=(r, port, out)) for r in range(2)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(120)
        assert all(p.exitcode == 0 for p in ps)
        assert dict(out) == {0: 5, 1: 5}
    assert bench._agree_max(7, None) == 7
