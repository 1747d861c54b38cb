"""The one-CTA bf16 grouped GEMM (used when CTA pairs are switched off with
MOE_GEMM_PAIR=0) must pass the same parity checks as the CTA-pair kernel
that runs by default.  Runs the bf16 parity cases in a child process."""
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_one_cta_bf16_gemm_parity():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, MOE_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_gpu_parity.py", "-m", "gpu", "-q",
                        "-k", "bf16", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
