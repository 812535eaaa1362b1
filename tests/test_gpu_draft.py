"""Parity of the MTP drafter (spec_draft through the C ABI) with the oracle.

Each sequence's drafter inputs (target activation, last token) are redrawn
until every one of the k oracle draft steps has a safe top-2 margin; the
draft tokens must then be identical and their logits within 2e-2 absolute
+ 1e-2 relative.  The drafter only reads the target's cache: every pool
byte is unchanged afterwards.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import workloads as W
from speculative_decoding_verification_91_b200.runtime import DeviceDrafter, Workspace, to_device_bf16
from speculative_decoding_verification_91_b200.session import WorkloadSession

from . import harness

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    B.lib()
    yield
    torch.cuda.synchronize()


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def device_drafter(wl, clusters=None):
    dd, hq, _ = W.drafter_spec(wl)
    emb, down, upw, blocks = W.drafter_weights(wl)
    return DeviceDrafter(d_draft=dd, n_q_heads=hq, w_emb_bits=emb, w_down_bits=down,
                         w_up_bits=upw, blocks=blocks, clusters=clusters)


@pytest.mark.parametrize("name,k", [("tiny", 3), ("small_b1", 4), ("small_ragged", 3),
                                    ("small_b16", 2), ("small_b32", 2), ("small_loop", 5)])
def test_draft_matches_oracle(name, k):
    wl = W.get_workload(name)
    model = harness.oracle_model(wl)
    drafter = harness.oracle_drafter(wl)
    sess = WorkloadSession(wl)
    dev_dr = device_drafter(wl)
    Bn = wl.batch
    hidden = np.zeros((Bn, wl.d_model), np.uint16)
    toks = np.zeros(Bn, np.int32)
    want = []
    for b in range(Bn):
        L = int(sess.lens[b])
        caches = harness.context_caches(wl, model, b, 0, L)
        _, h_bits, tok, steps = harness.guarded_draft_inputs(wl, model, drafter, caches, b, L, k)
        hidden[b], toks[b] = h_bits, tok
        want.append(steps)
    pools = [p for ps in (sess.dm.k_pool, sess.dm.v_pool, sess.dm.ksb_pool) for p in ps if p is not None]
    before = [_bits(p).copy() for p in pools]
    ws = Workspace(B.spec_draft_workspace_bytes(sess.dm.desc, dev_dr.desc, Bn, sess.max_pages))
    drafts = torch.full((Bn * k,), -7, dtype=torch.int32, device="cuda")
    maxl = torch.zeros(Bn * k, dtype=torch.float32, device="cuda")
    B.spec_draft(sess.dm.desc, dev_dr.desc, sess.block_table, sess.max_pages, sess.seq_lens,
                 to_device_bf16(hidden, "cuda"), torch.from_numpy(toks).cuda(), Bn, k, drafts, maxl,
                 ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    got = drafts.cpu().numpy().reshape(Bn, k)
    got_max = maxl.cpu().numpy().reshape(Bn, k)
    for b in range(Bn):
        assert list(got[b]) == [st.token for st in want[b]], (b, got[b], [st.token for st in want[b]])
        np.testing.assert_allclose(got_max[b], [st.top1 for st in want[b]], atol=ATOL, rtol=RTOL)
    for bef, p in zip(before, pools):
        assert np.array_equal(bef, _bits(p))
    assert np.array_equal(sess.seq_lens.cpu().numpy(), sess.lens)


def test_draft_zero_steps_launches_nothing():
    wl = W.get_workload("tiny")
    sess = WorkloadSession(wl)
    dev_dr = device_drafter(wl)
    ws = Workspace(B.spec_draft_workspace_bytes(sess.dm.desc, dev_dr.desc, 1, sess.max_pages))
    n0 = B.spec_launch_count()
    B.spec_draft(sess.dm.desc, dev_dr.desc, sess.block_table, sess.max_pages, sess.seq_lens,
                 torch.zeros(wl.d_model, dtype=torch.bfloat16, device="cuda"),
                 torch.zeros(1, dtype=torch.int32, device="cuda"), 1, 0,
                 torch.zeros(1, dtype=torch.int32, device="cuda"), None, ws.buf, ws.nbytes)
    assert B.spec_launch_count() == n0
