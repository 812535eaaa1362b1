"""The LM head + argmax entry point that allocates nothing.

Some callers cannot hand the library a workspace (a runtime whose device
memory plan is fixed before decoding, a plugin that only receives its input
and output tensors, a loop that cannot take cudaMalloc's implicit device
synchronisation).  spec_lmhead_argmax_noalloc serves them from a fixed
device array inside the library.  This file is collected last on purpose:
if it fails, a run that stops at the first failure has already run every
other test.  It passes alone in a fresh process (its first call performs the
per-device set-up) and after the other tests.

Its ids and maximum logits are checked against the oracle (margin-guarded
rows, as for spec_lmhead_argmax), and on two calls in a row against the
workspace entry point.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import gen
from speculative_decoding_verification_91_b200.runtime import Workspace, to_device_bf16

from . import harness

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 1e-2


def _case(tag, M, d, V):
    h = gen.normal_bf16(5, f"test/noalloc/{tag}/h", 0, M * d, 1.0).reshape(M, d)
    w = gen.normal_bf16(5, f"test/noalloc/{tag}/w", 0, V * d, 0.02).reshape(V, d)
    return h, w


# a: the b1_ctx8k LM head (5 rows, streaming kernel); b: 40 rows (tensor-memory
# kernel); c: the row limit, 64 rows
@pytest.mark.parametrize("tag,M,d,V", [("a", 5, 2560, 262144), ("b", 40, 1024, 9000),
                                       ("c", 64, 768, 5000)])
def test_noalloc_matches_oracle_and_workspace_entry_point(tag, M, d, V):
    assert torch.cuda.is_available()
    h, w = _case(tag, M, d, V)
    ids_o, t1, t2 = oracle.lm_head_top2(oracle.bf16_from_bits(h), w)
    hd, wd = to_device_bf16(h, "cuda"), to_device_bf16(w, "cuda")
    ws = Workspace(B.spec_lmhead_workspace_bytes(M, V))
    ids_ref = torch.zeros(M, dtype=torch.int32, device="cuda")
    max_ref = torch.zeros(M, dtype=torch.float32, device="cuda")
    B.spec_lmhead_argmax(hd, wd, M, d, V, ids_ref, max_ref, ws.buf, ws.nbytes)
    hv = oracle.bf16_from_bits(h).astype(np.float64)
    wv = oracle.bf16_from_bits(w).astype(np.float64)
    for call in range(2):                  # the array keeps the first call's contents
        ids = torch.full((M,), -7, dtype=torch.int32, device="cuda")
        mx = torch.zeros(M, dtype=torch.float32, device="cuda")
        B.spec_lmhead_argmax_noalloc(hd, wd, M, d, V, ids, mx)
        torch.cuda.synchronize()
        gi, gm = ids.cpu().numpy(), mx.cpu().numpy()
        for m in range(M):
            assert abs(gm[m] - t1[m]) <= ATOL + RTOL * abs(t1[m]), (tag, call, m)
            if harness.margin_ok(t1[m], t2[m]):
                assert gi[m] == ids_o[m], (tag, call, m, gi[m], ids_o[m])
            else:                          # a near tie: the pick must be a valid maximum
                assert 0 <= gi[m] < V
                assert abs(hv[m] @ wv[gi[m]] - t1[m]) <= ATOL + RTOL * abs(t1[m])
        # the same kernels as the workspace entry point: the same bits
        assert np.array_equal(gi, ids_ref.cpu().numpy()), (tag, call)
        assert np.array_equal(gm.view(np.uint32), max_ref.cpu().numpy().view(np.uint32)), (tag, call)
    assert B.spec_noalloc_read_status() == 0
    assert ws.device_status() == 0


def test_noalloc_status_bits_accumulate_until_read():
    """Device-detected errors of the workspace-free call are readable: bits set
    on the device (here injected from the host) survive later calls and are
    returned, then cleared, by spec_noalloc_read_status."""
    M, d, V = 5, 512, 3000
    h, w = _case("s", M, d, V)
    hd, wd = to_device_bf16(h, "cuda"), to_device_bf16(w, "cuda")
    ids = torch.zeros(M, dtype=torch.int32, device="cuda")
    assert B.spec_noalloc_read_status() == 0
    B.spec_noalloc_inject_status(B.SPEC_DEV_TIMEOUT)
    B.spec_lmhead_argmax_noalloc(hd, wd, M, d, V, ids, None)
    v = ctypes_read_status()
    assert v == (B.SPEC_ETIMEOUT, B.SPEC_DEV_TIMEOUT)
    assert B.spec_noalloc_read_status() == 0          # cleared by the read
    B.spec_noalloc_inject_status(B.SPEC_DEV_BAD_PAGE)
    assert ctypes_read_status() == (B.SPEC_EDEVICE, B.SPEC_DEV_BAD_PAGE)


def ctypes_read_status():
    """(return code, bits) of the C call itself."""
    import ctypes
    v = ctypes.c_uint(0)
    rc = B.lib().spec_noalloc_read_status(None, ctypes.byref(v))
    return rc, int(v.value)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    h, w = _case("r", 65, 64, 1000)
    hd, wd = to_device_bf16(h, "cuda"), to_device_bf16(w, "cuda")
    ids = torch.zeros(65, dtype=torch.int32, device="cuda")
    with pytest.raises(B.SpecError) as e:
        B.spec_lmhead_argmax_noalloc(hd, wd, 65, 64, 1000, ids, None)
    assert e.value.status == B.SPEC_EUNSUPPORTED
