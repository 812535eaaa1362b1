"""The tcgen05 split-KV attention kernel (opt-in through SPECVERIFY_TC_ATTN=1)
against the oracle: the attention-level and whole-step parity tests run
again in a child process with the tensor-memory path switched on."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_tc_attention_parity():
    env = dict(os.environ, SPECVERIFY_TC_ATTN="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_kernels.py"),
                        "-k", "verify_attn or verify_step or invariant"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
