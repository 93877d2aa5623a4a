"""The persistent single-row token-decoder step (PHOTON_STACK_MEGA=1) gives the
same results as the multi-kernel path: run in a child process with the switch
set (the library reads it once per process), small bf16 model, both modes."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_small_bf16_parity_with_persistent_token_steps():
    env = dict(os.environ, PHOTON_STACK_MEGA="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity_small_bf16.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
