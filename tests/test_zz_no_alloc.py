"""The LM head + argmax entry point that allocates nothing.

Some callers cannot hand the library a workspace (a runtime whose device
memory plan is fixed before decoding, a plugin that only receives its input
and output tensors, a loop that cannot take cudaMalloc's implicit device
synchronisation).  spec_lmhead_argmax_noalloc serves them from a fixed
device array inside the library.  This file is collected last on purpose:
if it fails, a run that stops at the first failure has already run every
other test.  It passes alone in a fresh process (its first call performs the
per-device set-up) and after the other tests.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import gen
from speculative_decoding_verification_91_b200.runtime import Workspace, to_device_bf16

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 1e-2


def _case(tag, M, d, V):
    h = gen.normal_bf16(5, f"test/noalloc/{tag}/h", 0, M * d, 1.0).reshape(M, d)
    w = gen.normal_bf16(5, f"test/noalloc/{tag}/w", 0, V * d, 0.02).reshape(V, d)
    return to_device_bf16(h, "cuda"), to_device_bf16(w, "cuda")


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    for tag, (M, d, V) in [("a", (5, 2560, 262144)), ("b", (64, 1024, 9000))]:
        hd, wd = _case(tag, M, d, V)
        ws = Workspace(B.spec_lmhead_workspace_bytes(M, V))
        ids_ref = torch.zeros(M, dtype=torch.int32, device="cuda")
        max_ref = torch.zeros(M, dtype=torch.float32, device="cuda")
        B.spec_lmhead_argmax(hd, wd, M, d, V, ids_ref, max_ref, ws.buf, ws.nbytes)
        ids = torch.zeros(M, dtype=torch.int32, device="cuda")
        mx = torch.zeros(M, dtype=torch.float32, device="cuda")
        B.spec_lmhead_argmax_noalloc(hd, wd, M, d, V, ids, mx)
        torch.cuda.synchronize()
        ref_v = max_ref.cpu().numpy()
        assert np.array_equal(ids.cpu().numpy(), ids_ref.cpu().numpy()), tag
        assert np.all(np.abs(mx.cpu().numpy() - ref_v) <= ATOL + RTOL * np.abs(ref_v)), tag


def test_noalloc_rejects_sizes_beyond_its_scratch():
    hd, wd = _case("c", 65, 64, 1000)
    ids = torch.zeros(65, dtype=torch.int32, device="cuda")
    with pytest.raises(B.SpecError) as e:
        B.spec_lmhead_argmax_noalloc(hd, wd, 65, 64, 1000, ids, None)
    assert e.value.status == B.SPEC_EUNSUPPORTED
