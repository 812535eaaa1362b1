"""Oracle of the MTP drafter's forward on the target's shared KV cache.

TEST INFRASTRUCTURE ONLY (see the package docstring).  numpy float64 with
bf16 / binary32 rounding at the points the model stores values in those
formats, as in `verify.py`.

Pages this follows (title and section):

[P1] "Gemma 4 拆解 | 多模态怎么塞进端侧，MTP drafter 又是怎么自带投机采样的"
     §4.2: the drafter's input is the target's last-layer activation of the
     previous step together with the embedding of the previous token (its
     own embedder); the two are concatenated and projected down to the
     drafter width; four blocks (three sliding-window, one global) attend to
     the target's KV cache instead of keeping a cache of their own, so the
     drafter needs no prefill and any draft length works; the result is
     projected back up to the target width and the target's unembedding
     picks the next draft token; k tokens are drafted autoregressively.
     §4.2 (figure): the blocks attend to the target's last prefilled local
     and global layers.
     §4.3: for small drafters the projection onto the whole vocabulary is
     replaced by a top-k over token clusters: the clusters' centroids are
     scored first and only the tokens of the best clusters (~4096) get real
     logits.
[P5] "Gemma 4 与 Gemini Nano：端侧智能的架构拆解" §草稿模型: the drafter reuses
     the base model's KV cache.

Readings where the pages leave a step open (the pages omit RoPE, norms and
the block internals from their sketch):
  * a block is x <- x + W_o CrossAttn(RMSNorm(x)), the shape of the
    target's own synthetic layers (no MLP); RMSNorm eps and unit gain as
    the target's;
  * the block's queries (n_q_heads heads of the target's head_dim) read the
    cache of one target layer as it is stored (post-RoPE keys; values, or
    pre-RoPE keys on key-equals-value layers), query head h reading KV head
    h // (n_q_heads / n_kv_heads); the query is rotated like that layer's
    keys (RoPE or p-RoPE) at its own position;
  * draft step s (0-based) of a sequence with committed length L sits at
    position L + s: the token it reads (the last accepted token at s = 0,
    its own previous draft after that) is the one at that position.  The
    cache holds positions < L only (the drafter writes nothing), so key j is
    visible iff j < L, and on a window-W block also j > L + s - W.  A query
    that sees no key gets a zero attention output;
  * the concatenation order is [target activation, token embedding]; every
    projection reads bf16 (the activation and the residual stream are
    rounded to bf16 where they enter a projection, as the target's GEMM
    inputs are); the up-projection's output (binary32) is both the next
    step's activation and, after the target's final RMSNorm (rounded to
    bf16), the input of the target's LM head; argmax ties go to the lowest
    token id;
  * cheap unembedding: every token belongs to exactly one cluster; a
    cluster's logit is h . centroid with the centroid a bf16 row of the
    tables; the n_select best clusters are kept (ties: lower cluster id);
    their tokens are scored with the target's LM-head rows and the argmax
    over those candidates is the draft token (ties: lowest token id).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .verify import (LayerCache, Model, attend, bf16, bf16_from_bits, f32, lm_head_top2, rmsnorm,
                     rope)

__all__ = ["DraftBlockDef", "Drafter", "ClusterTables", "cheap_unembed", "cross_attention",
           "draft_step", "draft"]


@dataclass
class DraftBlockDef:
    target_layer: int            # target layer whose cache this block reads
    w_q: np.ndarray              # float32 values [n_q_heads * D][d_draft]
    w_o: np.ndarray              # float32 values [d_draft][n_q_heads * D]


@dataclass
class Drafter:
    d_draft: int
    n_q_heads: int
    w_emb_bits: np.ndarray       # [V][d_draft] bf16 bits: the drafter's own embedder
    w_down: np.ndarray           # float32 values [d_draft][d_model + d_draft]
    w_up: np.ndarray             # float32 values [d_model][d_draft]
    blocks: list                 # DraftBlockDef, in order


def cross_attention(model: Model, drafter: Drafter, blk: DraftBlockDef, cache: LayerCache, L: int,
                    pos: int, q_pre) -> np.ndarray:
    """Attention of one drafter query (all heads) over a target layer's cache.

    q_pre [n_q_heads][D] binary32 values before RoPE; the query is rotated
    at `pos` with the target layer's RoPE fraction and rounded to bf16.  The
    cache holds positions [cache.lo, L).  Returns bf16 values [n_q_heads][D]."""
    spec = model.layers[blk.target_layer]
    D, Hkv = model.head_dim, model.n_kv_heads
    if cache.end != L:
        raise ValueError("cache does not end at the committed length")
    q_rot = bf16(rope(np.asarray(q_pre, dtype=np.float32)[None], [pos], D, model.rope_theta,
                      spec.rope_fraction))[0]
    kpos = np.arange(cache.lo, L)
    vis = kpos <= pos
    if spec.window > 0:
        vis &= kpos > pos - spec.window
    G = drafter.n_q_heads // Hkv
    out = np.zeros((drafter.n_q_heads, D), dtype=np.float64)
    if not vis.any():
        return bf16(out)
    keys, vals = cache.k[vis], cache.values()[vis]
    scale = 1.0 / np.sqrt(D)
    for h in range(drafter.n_q_heads):
        kh = h // G
        out[h] = attend(q_rot[h][None], keys[:, kh, :], vals[:, kh, :], [pos], kpos[vis],
                        spec.window, scale)[0]
    return bf16(out)


@dataclass
class ClusterTables:
    """Token clusters for the cheap unembedding ([P1] §4.3).

    cluster_tokens [C][S]: token ids of each cluster (-1 pads a short last
    cluster; every token sits in exactly one cluster); centroids_bits
    [C][d_model] bf16 bits; n_select: clusters whose tokens are scored."""
    cluster_tokens: np.ndarray
    centroids_bits: np.ndarray
    n_select: int


def cheap_unembed(h, w_lm_bits, tables: ClusterTables):
    """Argmax over the tokens of the best-scoring clusters instead of the
    whole vocabulary ([P1] §4.3 `cheap_unembed`).

    h [M][d] (bf16 values).  Each cluster logit is h . centroid (float64,
    rounded to binary32); the n_select clusters with the largest logits are
    kept (equal logits: lower cluster id first); every token of those
    clusters gets its logit h . W_v (float64, rounded to binary32) and the
    largest wins (equal logits: lowest token id).  Returns (ids [M], top1
    [M], top2 [M]) over the candidates."""
    h = np.asarray(h, dtype=np.float64)
    cent = bf16_from_bits(tables.centroids_bits).astype(np.float64)
    C = cent.shape[0]
    M = h.shape[0]
    ids = np.zeros(M, dtype=np.int64)
    top1, top2 = np.zeros(M), np.zeros(M)
    for m in range(M):
        cl = f32(h[m] @ cent.T).astype(np.float64)
        order = sorted(range(C), key=lambda c: (-cl[c], c))
        sel = order[:tables.n_select]
        cand = np.sort(np.concatenate([tables.cluster_tokens[c] for c in sel]))
        cand = cand[cand >= 0]
        lg = f32(h[m] @ bf16_from_bits(w_lm_bits[cand]).astype(np.float64).T).astype(np.float64)
        j = int(np.argmax(lg))                 # first maximum: candidates are in id order
        ids[m], top1[m] = cand[j], lg[j]
        rest = np.delete(lg, j)
        top2[m] = rest.max() if rest.size else -np.inf
    return ids, top1, top2


@dataclass
class DraftStep:
    h: np.ndarray                # up-projection output (binary32) [d_model]
    token: int                   # argmax of the target's LM head on RMSNorm(h)
    top1: float
    top2: float


def draft_step(model: Model, drafter: Drafter, caches: list, L: int, s: int, prev_hidden,
               prev_token: int, tables: ClusterTables | None = None) -> DraftStep:
    """One drafter forward ([P1] §4.2 `draft_one_step`) at position L + s; the
    draft token comes from the full LM head, or from the cheap clustered
    unembedding ([P1] §4.3) when cluster tables are given."""
    D = model.head_dim
    tok = bf16_from_bits(drafter.w_emb_bits[int(prev_token)]).astype(np.float64)
    u = np.concatenate([bf16(prev_hidden).astype(np.float64), tok])
    x = f32(u @ drafter.w_down.astype(np.float64).T)
    for blk in drafter.blocks:
        hn = bf16(rmsnorm(x, model.rms_eps)).astype(np.float64)
        q_pre = f32(hn @ blk.w_q.astype(np.float64).T).reshape(drafter.n_q_heads, D)
        o = cross_attention(model, drafter, blk, caches[blk.target_layer], L, L + s, q_pre)
        y = f32(o.reshape(-1).astype(np.float64) @ blk.w_o.astype(np.float64).T)
        x = f32(x.astype(np.float64) + y.astype(np.float64))
    h = f32(bf16(x).astype(np.float64) @ drafter.w_up.astype(np.float64).T)
    hn = bf16(rmsnorm(h, model.rms_eps))
    if tables is None:
        g, t1, t2 = lm_head_top2(hn[None], model.w_lm_bits)
    else:
        g, t1, t2 = cheap_unembed(hn[None], model.w_lm_bits, tables)
    return DraftStep(h, int(g[0]), float(t1[0]), float(t2[0]))


def draft(model: Model, drafter: Drafter, caches: list, L: int, prev_hidden, prev_token: int,
          k: int, tables: ClusterTables | None = None) -> list:
    """k autoregressive drafter steps ([P1] §4.2 `draft`): step s reads the
    previous step's up-projection output and draft token.  Returns the list
    of DraftStep."""
    out = []
    hidden, tok = np.asarray(prev_hidden, dtype=np.float32), int(prev_token)
    for s in range(k):
        st = draft_step(model, drafter, caches, L, s, hidden, tok, tables)
        out.append(st)
        hidden, tok = st.h, st.token
    return out
