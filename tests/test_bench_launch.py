"""bench.py's multi-rank launch on CPU (gloo, no GPU work).

`bench.py --gpus N` without a torchrun environment must start N ranks itself,
and under torchrun it must use the ranks it is given; either way the ranks
sum a replicated-gradient set through the same fp32 bucket the GPU run uses
and rank 0 prints one JSON line with the real world size.  The reference arm
(the CPU oracle on a bounded sample) must print its line too.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(cmd, timeout=240):
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout, env=env)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("n", [2, 3])
def test_gpus_n_launches_n_ranks(n):
    d = _run([sys.executable, "bench.py", "--gpus", str(n), "--plumbing-check"])
    assert d == {"plumbing_check": "ok", "n_gpus": n, "ranks": n, "backend": "gloo"}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_torchrun_ranks_are_used():
    d = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
              "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
              "--plumbing-check"])
    assert d["n_gpus"] == 2 and d["plumbing_check"] == "ok"


def test_reference_arm_line():
    d = _run([sys.executable, "bench.py", "--impl", "reference", "--config", "C1", "--steps", "1", "--warmup", "3"])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
