"""The bench's N > 1 path on the host: two gloo ranks launched by torchrun the
way the multi-GPU bench is launched (127.0.0.1 rendezvous), checking the
max-over-ranks timing, the weak-scaling aggregate, per-rank inputs and that
the oracle arm prints exactly one line, from rank 0."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun(n, *argv, timeout=240):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), *argv]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)
    lines = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]
    return p, lines


def test_two_rank_max_and_aggregate(tmp_path):
    p, _ = torchrun(2, "tests/dist_worker.py", "2", str(tmp_path))
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads((tmp_path / ("rank%d.json" % r)).read_text()) for r in range(2)]
    by_rank = {x["rank"]: x for x in lines}
    assert sorted(by_rank) == [0, 1]
    for x in by_rank.values():
        assert x["world"] == 2
        assert x["slowest_ms"] == 15.0                  # max over ranks, seen by every rank
        assert x["value"] == pytest.approx(2 * 2e12 / 15e-3 / 1e12)
    assert by_rank[0]["seed"] != by_rank[1]["seed"]     # independent inputs per rank
    assert {x["local"] for x in lines} == {0, 1}


def test_world_size_mismatch_is_refused():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, "tests/dist_worker.py", "2", "."], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=120)
    assert p.returncode != 0
    assert "WORLD_SIZE=1" in p.stderr


def test_reference_arm_two_ranks_prints_once():
    p, lines = torchrun(2, "bench.py", "--impl", "reference", "--gpus", "2", "--config", "lowres",
                        "--steps", "1", "--warmup", "3", timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
