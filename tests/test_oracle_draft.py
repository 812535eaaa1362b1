"""Pins of the drafter oracle (CPU only).

The drafter's cross-attention is checked against torch's scaled-dot-product
attention with an explicit visibility mask, its position convention by the
window edge (one visible key gives that key's value exactly, none gives
zero), the input concatenation and projections against torch's linear
layers in the degenerate case where every block adds nothing, and the
autoregressive loop against single steps.
"""
import copy

import numpy as np
import pytest
import torch

from oracle import draft as OD
from oracle import verify as OV

D, HKV, HQD, DM, DD, V = 16, 2, 4, 32, 16, 50


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bits(x):
    return OV.bits_from_bf16(x)


def _model(window, kv_equal, frac, seed=0):
    r = _rng(seed)
    layer = OV.LayerDef(window, kv_equal, frac, np.zeros((1, DM), np.float32),
                        np.zeros((DM, 1), np.float32))
    return OV.Model(DM, 4, HKV, D, _bits(r.standard_normal((V, DM)) * 0.3), [layer])


def _cache(model, L, seed=1):
    r = _rng(seed)
    spec = model.layers[0]
    k_raw = OV.bf16(r.standard_normal((L, HKV, D)))
    v_raw = None if spec.kv_equal else OV.bf16(r.standard_normal((L, HKV, D)))
    return OV.cache_from_raw(model, 0, 0, k_raw, v_raw)


def _drafter(seed=2, zero_o=False, n_blocks=2):
    r = _rng(seed)
    blocks = []
    for _ in range(n_blocks):
        w_q = OV.bf16(r.standard_normal((HQD * D, DD)) * 0.3)
        w_o = OV.bf16(r.standard_normal((DD, HQD * D)) * 0.1)   # drawn either way: same stream
        blocks.append(OD.DraftBlockDef(0, w_q, np.zeros_like(w_o) if zero_o else w_o))
    return OD.Drafter(DD, HQD, _bits(r.standard_normal((V, DD))),
                      OV.bf16(r.standard_normal((DD, DM + DD)) * 0.2),
                      OV.bf16(r.standard_normal((DM, DD)) * 0.3), blocks)


def _sdpa(q, k, v, mask, scale):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=torch.from_numpy(mask)[None, None], scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("window,kv_equal,frac,s", [(0, False, 1.0, 0), (0, True, 0.25, 2),
                                                    (7, False, 1.0, 0), (7, False, 1.0, 3),
                                                    (12, True, 0.25, 1)])
def test_cross_attention_is_masked_sdpa(window, kv_equal, frac, s):
    model, L = _model(window, kv_equal, frac), 20
    cache, dr = _cache(model, L), _drafter()
    q_pre = OV.f32(_rng(5).standard_normal((HQD, D)))
    pos = L + s
    got = OD.cross_attention(model, dr, dr.blocks[0], cache, L, pos, q_pre)
    q_rot = OV.bf16(OV.rope(q_pre[None], [pos], D, model.rope_theta, frac))[0]
    kpos = np.arange(L)
    mask = (kpos <= pos) & ((kpos > pos - window) if window else True)
    G = HQD // HKV
    for h in range(HQD):
        want = _sdpa(q_rot[h][None], cache.k[:, h // G], cache.values()[:, h // G], mask[None],
                     1.0 / np.sqrt(D))[0]
        np.testing.assert_array_equal(got[h], OV.bf16(want))


def test_query_position_is_committed_length_plus_step():
    # window 3, cache positions 0..4 (L = 5): step 1 sits at 6 and sees only
    # key 4, so its output is that key's value exactly; step 0 (position 5)
    # also sees key 3
    model, L = _model(3, False, 1.0), 5
    cache, dr = _cache(model, L), _drafter()
    q_pre = OV.f32(_rng(6).standard_normal((HQD, D)))
    out1 = OD.cross_attention(model, dr, dr.blocks[0], cache, L, L + 1, q_pre)
    G = HQD // HKV
    for h in range(HQD):
        np.testing.assert_array_equal(out1[h], cache.v[4, h // G])
    out0 = OD.cross_attention(model, dr, dr.blocks[0], cache, L, L, q_pre)
    assert not np.array_equal(out0, out1)


def test_no_visible_key_gives_zero():
    model, L = _model(1, False, 1.0), 6       # window 1 at position L + 1: nothing cached
    cache, dr = _cache(model, L), _drafter()
    out = OD.cross_attention(model, dr, dr.blocks[0], cache, L, L + 1,
                             OV.f32(_rng(7).standard_normal((HQD, D))))
    assert np.array_equal(out, np.zeros_like(out))


def test_projections_and_unembed_when_blocks_add_nothing():
    # every W_o = 0: h = W_up bf16(W_down [bf16(prev) || emb(tok)]) and the draft
    # is the LM head's argmax on RMSNorm(h); torch linear layers, rms_norm
    # and argmax give the same
    model, L = _model(0, False, 1.0), 9
    cache, dr = _cache(model, L), _drafter(zero_o=True)
    prev = OV.f32(_rng(8).standard_normal(DM))
    tok = 17
    st = OD.draft_step(model, dr, [cache], L, 0, prev, tok)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    u = torch.cat([t(OV.bf16(prev)), t(OV.bf16_from_bits(dr.w_emb_bits[tok]))])
    x = torch.nn.functional.linear(u, t(dr.w_down)).float()
    h = torch.nn.functional.linear(x.to(torch.bfloat16).double(), t(dr.w_up)).float()
    np.testing.assert_array_equal(st.h, h.numpy())
    hn = torch.nn.functional.rms_norm(h.double(), (DM,), eps=model.rms_eps)
    hn = hn.float().to(torch.bfloat16).double()
    logits = torch.nn.functional.linear(hn, t(OV.bf16_from_bits(model.w_lm_bits))).float()
    assert st.token == int(torch.argmax(logits))
    assert st.top1 == pytest.approx(float(logits.max()), rel=1e-6)


def test_draft_is_autoregressive_and_reads_only():
    model, L = _model(7, True, 0.25), 15
    cache, dr = _cache(model, L), _drafter(n_blocks=3)
    before = copy.deepcopy(cache)
    prev = OV.f32(_rng(9).standard_normal(DM))
    steps = OD.draft(model, dr, [cache], L, prev, 3, 4)
    assert len(steps) == 4
    hidden, tok = prev, 3
    for s, st in enumerate(steps):
        one = OD.draft_step(model, dr, [cache], L, s, hidden, tok)
        assert one.token == st.token and np.array_equal(one.h, st.h)
        hidden, tok = one.h, one.token
    shorter = OD.draft(model, dr, [cache], L, prev, 3, 2)
    assert [x.token for x in shorter] == [x.token for x in steps[:2]]
    assert OD.draft(model, dr, [cache], L, prev, 3, 0) == []
    for a, b in ((cache.k, before.k), (cache.kpre, before.kpre)):
        assert np.array_equal(a, b)


def test_draft_step_queries_sit_at_L_plus_s():
    # window 2: step 2 sits at L + 2 and no cached key (< L) is in its window,
    # so its blocks add nothing and it equals the same drafter with W_o = 0;
    # step 0 (position L) sees key L - 1 and does not
    model, L = _model(2, False, 1.0), 11
    cache = _cache(model, L)
    dr, dr0 = _drafter(seed=4), _drafter(seed=4, zero_o=True)
    prev = OV.f32(_rng(10).standard_normal(DM))
    a2 = OD.draft_step(model, dr, [cache], L, 2, prev, 5)
    b2 = OD.draft_step(model, dr0, [cache], L, 2, prev, 5)
    assert np.array_equal(a2.h, b2.h)
    a0 = OD.draft_step(model, dr, [cache], L, 0, prev, 5)
    b0 = OD.draft_step(model, dr0, [cache], L, 0, prev, 5)
    assert not np.array_equal(a0.h, b0.h)


# ---------------------------------------------------------------- cheap unembedding

def _tables(V, S, d, n_select, seed=3):
    r = _rng(seed)
    perm = r.permutation(V)
    C = -(-V // S)
    toks = np.full((C, S), -1, np.int64)
    toks.reshape(-1)[:V] = perm
    cent = _bits(r.standard_normal((C, d)))
    return OD.ClusterTables(toks, cent, n_select)


def test_cheap_unembed_over_every_cluster_is_the_full_argmax():
    r = _rng(11)
    V, d = 1000, 24
    w = _bits(r.standard_normal((V, d)))
    h = OV.bf16(r.standard_normal((5, d)))
    t = _tables(V, 16, d, n_select=-(-V // 16))
    ids, t1, _ = OD.cheap_unembed(h, w, t)
    fids, ft1, _ = OV.lm_head_top2(h, w)
    assert np.array_equal(ids, fids) and np.array_equal(t1, ft1)


@pytest.mark.parametrize("n_select", [1, 3, 7])
def test_cheap_unembed_keeps_the_best_clusters(n_select):
    # reference: cluster logits by torch matmul, kept set by a stable
    # lexicographic sort (logit descending, id ascending), argmax over the
    # kept tokens by torch (first maximum in token-id order)
    r = _rng(12 + n_select)
    V, S, d = 203, 8, 12          # 26 clusters, the last one 3 tokens short
    w = _bits(r.standard_normal((V, d)))
    t = _tables(V, S, d, n_select)
    t.centroids_bits[5] = t.centroids_bits[9]          # a tie between two clusters
    h = OV.bf16(r.standard_normal((6, d)))
    ids, t1, _ = OD.cheap_unembed(h, w, t)
    tt = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    cl = torch.nn.functional.linear(tt(h), tt(OV.bf16_from_bits(t.centroids_bits))).float().numpy()
    for m in range(h.shape[0]):
        order = np.lexsort((np.arange(cl.shape[1]), -cl[m].astype(np.float64)))
        cand = np.sort(t.cluster_tokens[order[:n_select]].reshape(-1))
        cand = cand[cand >= 0]
        lg = torch.nn.functional.linear(tt(h[m]), tt(OV.bf16_from_bits(w[cand]))).float()
        j = int(torch.argmax(lg))
        assert ids[m] == cand[j] and t1[m] == float(lg[j])


def test_cheap_unembed_tie_at_the_kept_boundary_keeps_the_lower_cluster_id():
    # clusters 5 and 9 share the same centroid, aligned with h, so they tie
    # for first place far above every other cluster; keeping one cluster
    # must keep cluster 5, and the argmax then lies among its tokens
    r = _rng(31)
    V, S, d = 203, 8, 12
    w = _bits(r.standard_normal((V, d)))
    t = _tables(V, S, d, n_select=1)
    h = OV.bf16(r.standard_normal((2, d)))
    for m in range(2):
        t.centroids_bits[5] = t.centroids_bits[9] = _bits(h[m] * 8.0)
        cent = OV.bf16_from_bits(t.centroids_bits).astype(np.float64)
        cl = cent @ h[m].astype(np.float64)
        assert cl[5] == cl[9] and np.sum(cl >= cl[5]) == 2       # the tie is for first place
        ids, _, _ = OD.cheap_unembed(h[m:m + 1], w, t)
        assert ids[0] in set(int(x) for x in t.cluster_tokens[5] if x >= 0)


def test_draft_step_with_clusters_uses_them():
    model, L = _model(0, False, 1.0), 9
    cache, dr = _cache(model, L), _drafter()
    prev = OV.f32(_rng(13).standard_normal(DM))
    full = OD.draft_step(model, dr, [cache], L, 0, prev, 4)
    every = OD.draft_step(model, dr, [cache], L, 0, prev, 4, _tables(V, 5, DM, n_select=V // 5))
    assert (every.token, every.top1) == (full.token, full.top1)
    one = OD.draft_step(model, dr, [cache], L, 0, prev, 4, _tables(V, 5, DM, n_select=1))
    assert np.array_equal(one.h, full.h)
