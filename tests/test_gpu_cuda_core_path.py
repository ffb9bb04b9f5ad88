"""The CUDA-core kernels (fp32 math everywhere) must match the oracle on the same
cases as the tensor-core kernels: the parity tests are re-run in a child process
with the tensor-core paths switched off."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_with_tensor_cores_disabled():
    env = dict(os.environ, CSA_B200_DISABLE_TC="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"), "-k", "small or tiny or ragged or topk"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
