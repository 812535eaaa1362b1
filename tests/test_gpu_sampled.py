"""Parity of sampled verification (spec_verify_step_sampled) with the oracle.

Draft logits are seeded synthetic inputs; the drafts are drawn from their
softmax with seeded uniforms, and the acceptance and draw uniforms are
seeded too.  A sequence's draws are redrawn (oracle only) until every
acceptance decision is at least 5% away from its threshold and the Gumbel
draw's winner leads by more than the logits' tolerance and is not a
near-cancellation of p - q; then accept lengths, emitted tokens, next token
and lengths must be identical, and the target logits within 2e-2 + 1e-2
relative."""
import numpy as np
import pytest
import torch

import oracle
from oracle import sampled as OS
from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import gen
from speculative_decoding_verification_91_b200.inputs import workloads as W
from speculative_decoding_verification_91_b200.runtime import Workspace
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


REL = 0.05   # relative error of p and q allowed for: the logits agree to 2e-2 (+1e-2 relative)


def _safe(res, pl, dl, g, T, k):
    """The decisions hold for any p, q within REL relative of the oracle's: each
    acceptance test is more than REL from its threshold, and the drawn
    token's lowest possible Gumbel score beats every other token's highest
    (the residual max(0, p - q) can grow from zero where p and q nearly
    cancel)."""
    if res.accept_margin < REL:
        return False
    a = res.accept_len
    p = OS.softmax(pl[a], T)
    q = OS.softmax(dl[a], T) if a < k else np.zeros_like(p)
    gum = -np.log(-np.log(np.asarray(g, dtype=np.float64)))
    slack = REL * np.maximum(p, q)
    w = np.maximum(p - q, 0.0)
    t = res.next_last_token
    w_lo = w[t] - slack[t]
    if w_lo <= 0:
        return False
    s_lo = np.log(w_lo) + gum[t]
    w_hi = w + slack
    s_hi = np.log(w_hi) + gum
    s_hi[t] = -np.inf
    return bool(s_hi.max() < s_lo)


def _case(wl, model, caches, L, last, b, k, T, name):
    """Draft i is drawn from q_i = softmax((the oracle target's logits of row i
    + seeded N(0, 0.3) noise) / T), row i seeing the drafts before it, so
    that drafts are often accepted; then the acceptance and draw uniforms."""
    V = wl.vocab
    for t in range(60):
        key = f"test/sampled/{name}/b{b}/a{t}"
        ud = gen.uniform(7, key + "/ud", 0, max(k, 1))
        drafts, dl = [], np.zeros((k, V), np.float32)
        for i in range(k):
            fw_i = oracle.verify_forward(model, caches, L, [last] + drafts, lm_rows=[i])
            noise = gen.normal_f32(7, key + f"/dl{i}", 0, V, 0.3)
            dl[i] = OS.full_logits(fw_i.h, model.w_lm_bits)[0] + noise
            q = OS.softmax(dl[i], T)
            drafts.append(int(min(np.searchsorted(np.cumsum(q), ud[i]), V - 1)))
        fw = oracle.verify_forward(model, caches, L, [last] + drafts)
        pl = OS.full_logits(fw.h, model.w_lm_bits)
        # the device reads binary32 uniforms: the oracle gets the same values
        ua = gen.uniform(7, key + "/ua", 0, max(k, 1))[:k].astype(np.float32)
        g = np.clip(gen.uniform(7, key + "/g", 0, V), 1e-7, 1 - 1e-7).astype(np.float32)
        res = OS.speculative_sample(pl, dl, drafts, ua, g, T)
        if _safe(res, pl, dl, g, T, k):
            return drafts, dl, ua, g, pl, res
    raise RuntimeError("no safe sampled case")


@pytest.mark.parametrize("name,T,k", [("small_b1", 1.0, 4), ("small_ragged", 0.8, 4),
                                      ("small_ragged", 1.0, 0), ("small_b32", 1.0, 3)])
def test_sampled_verify_matches_oracle(name, T, k):
    wl = W.get_workload(name)
    model = harness.oracle_model(wl)
    sess = WorkloadSession(wl)
    Bn, V, q = wl.batch, wl.vocab, k + 1
    drafts = np.zeros((Bn, max(k, 1)), np.int32)
    dls = np.zeros((Bn, max(k, 1), V), np.float32)
    uas = np.zeros((Bn, max(k, 1)), np.float32)
    gs = np.zeros((Bn, V), np.float32)
    lasts = np.zeros(Bn, np.int32)
    want, logits = [], []
    for b in range(Bn):
        L = int(sess.lens[b])
        caches = harness.context_caches(wl, model, b, 0, L)
        last = W.last_token(wl, b, 0)
        d, dl, ua, g, pl, res = _case(wl, model, caches, L, last, b, k, T, name)
        lasts[b] = last
        drafts[b, :k], dls[b, :k], uas[b, :k], gs[b] = d, dl, ua, g
        want.append(res)
        logits.append(pl)
    ws = Workspace(B.spec_verify_sampled_workspace_bytes(sess.dm.desc, Bn, k, sess.max_pages))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    acc = torch.zeros(Bn, dtype=torch.int32, device="cuda")
    emitted = torch.zeros(Bn * q, dtype=torch.int32, device="cuda")
    new_last = torch.zeros(Bn, dtype=torch.int32, device="cuda")
    tl = torch.zeros(Bn * q * V, dtype=torch.float32, device="cuda")
    B.spec_verify_step_sampled(sess.dm.desc, sess.block_table, sess.max_pages, dev(lasts),
                               dev(drafts[:, :k].reshape(-1)) if k else None,
                               dev(dls[:, :k].reshape(-1)) if k else None, Bn, k, T,
                               dev(uas[:, :k].reshape(-1)) if k else None, dev(gs.reshape(-1)),
                               sess.seq_lens, acc, emitted, new_last, tl, ws.buf, ws.nbytes)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    acc, emitted, new_last = acc.cpu().numpy(), emitted.cpu().numpy().reshape(Bn, q), new_last.cpu().numpy()
    tl = tl.cpu().numpy().reshape(Bn, q, V)
    for b in range(Bn):
        np.testing.assert_allclose(tl[b], logits[b], atol=ATOL, rtol=RTOL)
        assert acc[b] == want[b].accept_len, (b, acc[b], want[b].accept_len)
        assert list(emitted[b]) == want[b].emitted
        assert new_last[b] == want[b].next_last_token
    assert np.array_equal(sess.seq_lens.cpu().numpy(), sess.lens + acc + 1)
