"""Parity of the cheap clustered unembedding (spec_cluster_unembed, and the
drafter using it) with the oracle.  Rows whose oracle top-2 margin among
the candidates is within the float tolerance are skipped for the id check
(their logits are still compared); ids of the others must be identical."""
import numpy as np
import pytest
import torch

import oracle
from oracle import draft as OD
from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import gen
from speculative_decoding_verification_91_b200.inputs import workloads as W
from speculative_decoding_verification_91_b200.runtime import DeviceClusters, Workspace, to_device_bf16
from speculative_decoding_verification_91_b200.session import WorkloadSession

from . import harness
from .test_gpu_draft import device_drafter

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    B.lib()
    yield
    torch.cuda.synchronize()


def _tables(wl, w_lm=None, n_select=None):
    toks, cent, wc, ns = W.cluster_tables(wl, w_lm)
    ns = ns if n_select is None else n_select
    return (OD.ClusterTables(toks, cent, ns),
            DeviceClusters(cluster_tokens=toks, centroid_bits=cent, clustered_bits=wc, n_select=ns))


@pytest.mark.parametrize("name,M,n_select", [("small_b1", 1, None), ("small_b1", 12, None),
                                             ("small_b1", 40, 3), ("small_ragged", 7, 40),
                                             ("b1_ctx8k", 5, None)])
def test_cluster_unembed_matches_oracle(name, M, n_select):
    wl = W.get_workload(name)
    w_lm = W.lm_head_weight(wl)
    tables, dev = _tables(wl, w_lm, n_select)
    h_bits = gen.normal_bf16(5, f"test/cluster/{name}/{M}", 0, M * wl.d_model, 1.0).reshape(M, wl.d_model)
    h = oracle.bf16_from_bits(h_bits)
    ids, top1, top2 = OD.cheap_unembed(h, w_lm, tables)
    ws = Workspace(B.spec_cluster_unembed_workspace_bytes(M, wl.d_model, dev.desc))
    got = torch.full((M,), -5, dtype=torch.int32, device="cuda")
    gmax = torch.zeros(M, dtype=torch.float32, device="cuda")
    B.spec_cluster_unembed(to_device_bf16(h_bits, "cuda"), M, wl.d_model, dev.desc, got, gmax,
                           ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    got, gmax = got.cpu().numpy(), gmax.cpu().numpy()
    safe = np.array([harness.margin_ok(a, b) for a, b in zip(top1, top2)])
    assert safe.mean() >= 0.5, safe
    assert np.array_equal(got[safe], ids[safe]), (got, ids, safe)
    np.testing.assert_allclose(gmax, top1, atol=ATOL, rtol=RTOL)
    # a second call on the same workspace (keys were cleared) gives the same
    got2 = torch.zeros(M, dtype=torch.int32, device="cuda")
    B.spec_cluster_unembed(to_device_bf16(h_bits, "cuda"), M, wl.d_model, dev.desc, got2, None,
                           ws.buf, ws.nbytes)
    assert np.array_equal(got2.cpu().numpy(), got)


@pytest.mark.parametrize("name,k", [("small_b1", 4), ("small_ragged", 3)])
def test_draft_with_clusters_matches_oracle(name, k):
    wl = W.get_workload(name)
    model = harness.oracle_model(wl)
    drafter = harness.oracle_drafter(wl)
    tables, dev_cl = _tables(wl, model.w_lm_bits)
    sess = WorkloadSession(wl)
    dev_dr = device_drafter(wl, clusters=dev_cl)
    Bn = wl.batch
    hidden = np.zeros((Bn, wl.d_model), np.uint16)
    toks = np.zeros(Bn, np.int32)
    want = []
    for b in range(Bn):
        L = int(sess.lens[b])
        caches = harness.context_caches(wl, model, b, 0, L)
        _, h_bits, tok, steps = harness.guarded_draft_inputs(wl, model, drafter, caches, b, L, k,
                                                             tables=tables)
        hidden[b], toks[b] = h_bits, tok
        want.append(steps)
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
        assert list(got[b]) == [st.token for st in want[b]]
        np.testing.assert_allclose(got_max[b], [st.top1 for st in want[b]], atol=ATOL, rtol=RTOL)
