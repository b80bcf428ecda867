"""Concurrent host threads: the library keeps host-side caches (SM count,
per-device shared-memory attributes, the scratch address of the no-alloc
entry point) that every calling thread shares.  A fresh child process runs
ten threads that call prefill and decode at once on their own streams,
hitting the first launch of each kernel instance together, and checks every
result against the oracle."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_concurrent_host_threads_match_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    res = subprocess.run([sys.executable, "-m", "tests.threads_child"], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "threads ok" in res.stdout
