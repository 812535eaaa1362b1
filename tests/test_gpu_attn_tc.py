"""The two split-KV attention kernels against the oracle on every shape.

By default a layer without a sliding window takes the tcgen05 kernel when it
has at least four query heads per KV head, every other layer the mma.sync
kernel.  Here the attention-level, whole-step and k-invariance parity tests
run again in child processes with each kernel forced on for every layer
(head_dim 256): the tcgen05 kernel (SPECVERIFY_TC_ATTN_MIN_G=1 with
SPECVERIFY_TC_ATTN_LOCAL=1) and the mma.sync kernel (SPECVERIFY_NO_TC_ATTN=1)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
@pytest.mark.parametrize("env", [{"SPECVERIFY_TC_ATTN_MIN_G": "1", "SPECVERIFY_TC_ATTN_LOCAL": "1"},
                                 {"SPECVERIFY_NO_TC_ATTN": "1"}])
def test_attention_kernels_forced_parity(env):
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_kernels.py"),
                        "-k", "verify_attn or verify_step or invariant"],
                       cwd=ROOT, env=dict(os.environ, **env), capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
