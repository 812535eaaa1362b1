"""Test-side glue: turn a workload's seeded raw inputs into oracle objects and
into the drafts/expected outcomes the parity tests compare against.

Only tests (and the golden-fixture script) use this module; it imports the
oracle and the input generator, never the CUDA binding.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle
from speculative_decoding_verification_91_b200.inputs import workloads as W

MARGIN_ABS = 2e-2      # float tolerance of logits: 2e-2 absolute ...
MARGIN_REL = 1e-2      # ... plus 1e-2 relative


def margin_ok(top1: float, top2: float) -> bool:
    """Top-2 logit gap wider than the logits' float tolerance, so that any
    implementation within tolerance takes the same argmax."""
    return (top1 - top2) >= MARGIN_ABS + MARGIN_REL * abs(top1)


def oracle_model(wl: W.Workload) -> oracle.Model:
    layers = []
    for l, spec in enumerate(wl.layers):
        wqkv, wo = W.layer_weights(wl, l)
        layers.append(oracle.LayerDef(spec.window, spec.kv_equal, spec.rope_fraction,
                                      oracle.bf16_from_bits(wqkv), oracle.bf16_from_bits(wo)))
    return oracle.Model(wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                        W.lm_head_weight(wl), layers, wl.rope_theta, wl.rms_eps,
                        W.embedding_weight(wl))


def context_caches(wl: W.Workload, model: oracle.Model, b: int, attempt: int, L: int):
    caches = []
    for l in range(len(wl.layers)):
        lo, k, v = W.context_kv(wl, b, attempt, l, L)
        caches.append(oracle.cache_from_raw(model, l, lo, oracle.bf16_from_bits(k),
                                            None if v is None else oracle.bf16_from_bits(v)))
    return caches


def snapshot_caches(model: oracle.Model, pools, table_row, L: int, page: int = 64) -> list:
    """Oracle caches of one sequence rebuilt from the library's paged pools.

    pools[l] = (k_pool, v_pool or None, ksb_pool or None), each [P][Hkv][page][*]
    bf16 tensors (any device); table_row = the sequence's block-table row; L =
    its committed length.  Positions [lo, L) are gathered page by page, with
    lo = L - (window - 1) on sliding-window layers (0 on global ones).  On
    key-equals-value layers the values (the pre-RoPE keys) are the post-RoPE
    keys with their rotated dimensions taken from the side-band."""
    import torch
    out = []
    D = model.head_dim
    half = D // 2
    table_row = np.asarray(table_row)
    for l, spec in enumerate(model.layers):
        k_pool, v_pool, sb_pool = pools[l]
        lo = max(0, L - (spec.window - 1)) if spec.window > 0 else 0
        p0, p1 = lo // page, (L + page - 1) // page
        idx = torch.as_tensor(table_row[p0:p1].astype(np.int64), device=k_pool.device)

        def rows(pool):
            g = pool.index_select(0, idx)                          # [n_pages][Hkv][page][w]
            g = g.permute(0, 2, 1, 3).reshape(-1, pool.shape[1], pool.shape[3])
            bits = g[lo - p0 * page:L - p0 * page].contiguous().view(torch.int16).cpu().numpy()
            return oracle.bf16_from_bits(bits.view(np.uint16))

        k = rows(k_pool)
        if spec.kv_equal:
            n = sb_pool.shape[3] // 2
            sb = rows(sb_pool)
            kpre = k.copy()
            kpre[..., :n] = sb[..., :n]
            kpre[..., half:half + n] = sb[..., n:]
            out.append(oracle.LayerCache(lo, k, None, kpre))
        else:
            out.append(oracle.LayerCache(lo, k, rows(v_pool), None))
    return out


def greedy_continuation(model, caches, L, last, n):
    """First n greedy tokens after `last` (one oracle forward per token)."""
    toks = [int(last)]
    out = []
    for _ in range(n):
        fw = model_forward_last(model, caches, L, toks)
        out.append(int(fw.g[0]))
        toks.append(out[-1])
    return np.array(out, dtype=np.int64)


def model_forward_last(model, caches, L, toks):
    return oracle.verify_forward(model, caches, L, toks, lm_rows=[len(toks) - 1])


@dataclass
class SeqCase:
    b: int
    attempt: int
    L: int
    last: int
    drafts: np.ndarray
    r: int
    result: object          # oracle.StepResult
    guarded: bool           # rows 0..a all have a safe top-2 margin


def build_sequence(wl, model, b, L, attempt, guard=True) -> SeqCase:
    caches = context_caches(wl, model, b, attempt, L)
    last = W.last_token(wl, b, attempt)
    r = W.rejection_point(wl, b, attempt)
    n_greedy = wl.k if (r == wl.k or wl.accept[0] == "one_wrong") else r + 1
    greedy = greedy_continuation(model, caches, L, last, n_greedy)
    drafts, r2 = W.make_drafts(wl, b, attempt, np.concatenate([greedy, np.zeros(1, np.int64)]))
    assert r2 == r
    res = oracle.verify_step(model, caches, L, last, drafts)
    ok = res.accept_len == r and all(margin_ok(res.top1[i], res.top2[i])
                                     for i in range(res.accept_len + 1))
    return SeqCase(b, attempt, L, last, drafts, r, res, ok)


def guarded_sequence(wl, model, b, L, max_attempts=40, start=0) -> SeqCase:
    """Redraw the sequence's sub-seed (context, last token, drafts) until every
    argmax the acceptance depends on has a safe margin."""
    for t in range(start, start + max_attempts):
        case = build_sequence(wl, model, b, L, t)
        if case.guarded:
            return case
    raise RuntimeError(f"no margin-safe draw for sequence {b} in {max_attempts} attempts")


def oracle_drafter(wl: W.Workload):
    """The drafter of a workload as the oracle sees it (weights as values)."""
    from oracle import draft as OD
    dd, hq, _ = W.drafter_spec(wl)
    emb, down, upw, blocks = W.drafter_weights(wl)
    return OD.Drafter(dd, hq, emb, oracle.bf16_from_bits(down), oracle.bf16_from_bits(upw),
                      [OD.DraftBlockDef(t, oracle.bf16_from_bits(q), oracle.bf16_from_bits(o))
                       for q, o, t in blocks])


def guarded_draft_inputs(wl, model, drafter, caches, b, L, k, max_attempts=40, tables=None):
    """Redraw sequence b's drafter inputs (target activation, token) until every
    one of the k oracle draft steps has a safe top-2 margin.  Returns
    (attempt, activation bits, token, oracle steps)."""
    from oracle import draft as OD
    for t in range(max_attempts):
        h_bits, tok = W.drafter_inputs(wl, b, t)
        steps = OD.draft(model, drafter, caches, L, oracle.bf16_from_bits(h_bits), tok, k, tables)
        if all(margin_ok(st.top1, st.top2) for st in steps):
            return t, h_bits, tok, steps
    raise RuntimeError(f"no margin-safe drafter inputs for sequence {b}")
