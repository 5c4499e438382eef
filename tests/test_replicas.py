"""The N > 1 host path of bench.py on CPU (gloo, two ranks): every rank takes
the slowest rank's time, the whole-job rate counts all ranks' work, and the
reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_and_rate_with_two_gloo_ranks(tmp_path):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "_replica_worker.py")]
    env = dict(os.environ, OMP_NUM_THREADS="1", REPLICA_OUT=str(tmp_path))
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(2)]
    assert sorted(d["rank"] for d in lines) == [0, 1]
    slowest = max(d["local_ms"] for d in lines)
    for d in lines:
        assert d["world"] == 2
        assert d["ms"] == slowest
        assert abs(d["rate"] - 2 * 1000 / (slowest / 1e3)) < 1e-6


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""
