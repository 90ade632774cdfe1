"""bench.py's multi-GPU plumbing, on the CPU: two ranks launched the way the
driver launches the bench (torchrun, env:// rendezvous on 127.0.0.1), with
gloo in place of NCCL.  Each rank draws its own batch; the timings reduce
by max and the row counts by sum; the reference arm runs on rank 0 only."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from synthetic import workload_lengths  # noqa: E402


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_env() -> dict:
    env = dict(os.environ)
    env["CUDA_VISIBLE_DEVICES"] = ""
    env["MASTER_ADDR"] = "127.0.0.1"
    return env


def test_two_gloo_ranks(tmp_path):
    import bench
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
           os.path.join(ROOT, "tests", "ranks_worker.py"), str(tmp_path)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=240, env=_cpu_env(), cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    seen = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    wl = "ragged256_loguniform_1k_100k_d128_k64_bf16"
    rows = [int(workload_lengths(wl, bench.rank_seed(wl, i)).sum()) for i in range(2)]
    assert rows[0] != rows[1]  # each rank its own ragged batch
    for i, s in enumerate(seen):
        assert s["rank"] == i and s["world"] == 2
        assert s["rows"] == rows[i]
        assert s["rows_total"] == rows[0] + rows[1]
        assert s["max_time"] == 11.0  # the slowest rank's time
        assert s["sum_ranks"] == 3.0


def test_rank_seeds_differ_and_rank0_keeps_the_workload_seed():
    import bench
    from synthetic import WORKLOADS
    for name, w in WORKLOADS.items():
        assert bench.rank_seed(name, 0) == w.seed
        assert len({bench.rank_seed(name, r) for r in range(8)}) == 8


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank0_only(rank):
    env = _cpu_env()
    env.update({"RANK": str(rank), "WORLD_SIZE": "2", "LOCAL_RANK": str(rank)})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3",
                        "--workload", "batch32_n10k_d128_k64_bf16"],
                       capture_output=True, text=True, timeout=240, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    if rank != 0:
        assert r.stdout.strip() == ""
        return
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("impl", ["ours", "reference"])
def test_gpus_must_match_the_launched_ranks(impl):
    """--gpus 2 in a single process (no torchrun) is an error, not a silent
    one-GPU run reported as two; so is --gpus 1 among two ranks."""
    for gpus, world in ((2, None), (1, 2)):
        env = _cpu_env()
        for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
            env.pop(key, None)
        if world is not None:
            env.update({"RANK": "0", "WORLD_SIZE": str(world), "LOCAL_RANK": "0"})
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", impl,
                            "--gpus", str(gpus), "--steps", "1", "--warmup", "3",
                            "--workload", "batch32_n10k_d128_k64_bf16"],
                           capture_output=True, text=True, timeout=240, env=env, cwd=ROOT)
        assert r.returncode != 0 and "rank(s) were launched" in r.stderr, r.stderr[-1000:]
