"""The bench's host-side logic on the CPU.  The multi-GPU path is N
independent replicas (no collective on the data path): world_size-2 gloo
ranks exercise the process-group set-up from the torchrun environment, the
barrier, the max-over-ranks timing and the whole-job rate.  The reference
arm (the oracle on the host cores) runs on rank 0 only and prints the
contract's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_PROG = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import bench
import torch.distributed as dist
world, rank, local = bench.dist_setup(None)
assert (world, rank, local) == (2, int(os.environ["RANK"]), int(os.environ["LOCAL_RANK"]))
assert dist.get_backend() == "gloo"
bench.barrier(world)
ms = [3.0, 5.0][rank]                  # rank 1 is the slower one
ms_max = bench.max_over_ranks(world, ms)
rate = bench.whole_job_rate(world, 40, ms_max)
bench.barrier(world)
dist.destroy_process_group()
print(json.dumps({"rank": rank, "ms_max": ms_max, "rate": rate}))
"""


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch(args, world, port, extra_env=None):
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, *args], cwd=ROOT, env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            p.kill()
            out, err = p.communicate()
        outs.append((p.returncode, out, err))
    return outs


def test_two_gloo_ranks_barrier_max_and_rate():
    outs = launch(["-c", RANK_PROG, ROOT], 2, free_port())
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
    res = sorted((json.loads(o.strip().splitlines()[-1]) for _, o, _ in outs), key=lambda j: j["rank"])
    # every rank sees the slowest rank's time, and the rate counts both ranks' units
    assert [r["ms_max"] for r in res] == [5.0, 5.0]
    assert all(r["rate"] == pytest.approx(2 * 40 / 5e-3) for r in res)


def test_whole_job_rate_is_replicas_over_slowest():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_rate(1, 4 * 200, 10.0) == pytest.approx(80000.0)
    assert bench.whole_job_rate(8, 4 * 200, 10.0) == pytest.approx(8 * 80000.0)


def test_reference_arm_rank_nonzero_exits_without_work():
    """Under torchrun only rank 0 runs the reference arm; the others exit 0
    at once, print nothing and join no process group."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_reference_arm_json_line():
    """The reference arm times the oracle on the host cores and prints one
    JSON line with the native arm's metric, unit and workload, its own
    cpu_baseline and an end-to-end figure with no device copies."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.strip().splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference"
    assert j["metric"] == "decode MoE tokens/s" and j["unit"] == "tokens/s" and j["higher_is_better"]
    assert j["steps"] == 1 and j["warmup"] == 3 and j["value"] > 0
    assert "T=4" in j["config"]["workload"] and "d=2048" in j["config"]["workload"]
    assert j["config"]["tokens_per_step"] == 4 and j["config"]["same_window"] is True
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    assert cb["nproc"] >= 1 and cb["usable_cores"] == cb["cores"] and "cpu_model" in cb
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
