"""The NCCL paths (sequence sharding's all-gather, the data-parallel gradient
all-reduce) run for real with a world of one on cuda:0, in a child process so
that the process group does not outlive the test."""
import os
import socket
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_nccl_one_rank_paths():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()),
               RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, os.path.join(HERE, "_nccl_one_rank.py")], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-3000:])
    assert "nccl one-rank checks ok" in r.stdout
