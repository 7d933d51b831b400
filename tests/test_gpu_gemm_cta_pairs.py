"""The CTA-pair tiles of the tensor-core GEMM (256-row tiles over two SMs,
enabled with MO_GEMM_PAIR=1): the GEMM unit tests and Muon / SOAP parity
tests rerun in a child process with the switch set (it is read once per
process)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_cta_pair_tiles():
    env = dict(os.environ, MO_GEMM_PAIR="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(HERE, "test_gpu_gemm.py"),
           os.path.join(HERE, "test_gpu_muon.py") + "::test_dense_gpt_mini_buckets",
           os.path.join(HERE, "test_gpu_muon.py") + "::test_ragged_shapes_full_rank",
           os.path.join(HERE, "test_gpu_soap.py") + "::test_warm_step_parity"]
    r = subprocess.run(cmd, env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
