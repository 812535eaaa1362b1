"""Oracle: what one speculative-decoding verify step computes, written out plainly.

TEST INFRASTRUCTURE ONLY (see the package docstring).  numpy float64
arithmetic; values are rounded to bfloat16 or binary32 exactly where the
model stores them in those formats, and nowhere else.

Pages this follows (cited by title and section):

[P1] "Gemma 4 拆解 | 多模态怎么塞进端侧，MTP drafter 又是怎么自带投机采样的"
     §2 (global layers: p-RoPE with p = 0.25, value reuses key, global KV
     cache 37.5% smaller), §4.1 (the target checks k drafts in one forward;
     everything after the first wrong draft is cut), §4.2 (`speculative_step`:
     draft, `main_model.verify`, `accept_longest_prefix`; the drafter reads
     the target's KV cache).
[P2] "Accelerating Gemma 4: faster inference with multi-token prediction
     drafters" §3 (the target verifies the drafts in parallel, accepts the
     agreeing run and adds one token of its own).
[P3] "Gemma 4 发布时未包含 MTP 数据——为什么这很重要" §什么是 Gemma 4
     (alternating local sliding-window / global layers, p-RoPE, shared KV
     cache, key-equals-value), §什么是多标记预测 (drafts that agree with
     what the model would produce itself are accepted; generation falls back
     at the first wrong one), §MTP 能快多少 (the output is identical to
     standard decoding).

Readings where the pages leave a step open (each is a fixed convention of
this implementation):
  * acceptance is greedy: draft i is accepted iff it equals the target's
    argmax at that row;
  * rows i = 0..k carry [last_token, d_0..d_{k-1}] at positions L..L+k; the
    argmax of row i predicts position L+i+1;
  * attention scale 1/sqrt(D); no soft-cap, QK-norm or sinks; key j is
    visible to the query at position t iff j <= t and, on a window-W layer,
    j > t - W (W keys including itself);
  * RoPE pairs dimension i with i + D/2 (rotate-half), theta_i =
    base^(-2i/D), angle = position * theta_i; p-RoPE rotates only the pairs
    i < p*D/2 (the highest frequencies) and leaves the rest unchanged;
  * key-equals-value: V is the pre-RoPE key projection;
  * the synthetic target is x <- x + W_o Attn(RMSNorm(x)) per layer (no
    MLP), then RMSNorm and the LM head; RMSNorm eps 1e-6, unit gain; the
    token embedding is its own table (untied);
  * storage formats: fp32 residual stream; bf16 for normalised GEMM inputs,
    q/k/v after RoPE, cache entries, attention outputs and the final hidden
    state; logits in binary32; argmax ties go to the lowest token id.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "f32", "bf16", "bf16_from_bits", "bits_from_bf16",
    "rmsnorm", "rope_inv_freq", "rope_rotated_pairs", "rope_cos_sin", "rope",
    "attend", "lm_head_top2", "accept_longest_prefix",
    "LayerDef", "Model", "LayerCache", "cache_from_raw", "kv_values_per_token_head",
    "attention_layer", "verify_forward", "verify_step", "commit", "greedy_decode",
    "speculative_decode", "prefill",
]

# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------


def f32(x) -> np.ndarray:
    """Round to IEEE binary32 (round-to-nearest-even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16(x) -> np.ndarray:
    """Round to bfloat16, returned as float32 values.

    bfloat16 is the upper half of a binary32 pattern.  The value is first
    rounded to binary32 (the precision the kernels hold it in) and then to
    the nearest bfloat16, ties to even."""
    a = np.ascontiguousarray(f32(x))
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    r = np.where(np.isnan(a), np.uint32(0x7FC00000), r)
    return r.view(np.float32)


def bf16_from_bits(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def bits_from_bf16(x) -> np.ndarray:
    a = np.ascontiguousarray(bf16(x))
    return (a.view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------
# Elementwise pieces
# ---------------------------------------------------------------------------


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, unit gain (float64)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_inv_freq(head_dim: int, theta: float = 10000.0) -> np.ndarray:
    """theta_i = base^(-2i/D) for pairs i = 0..D/2-1 (float64)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / head_dim)


def rope_rotated_pairs(head_dim: int, fraction: float) -> int:
    """Number of rotated pairs: the first fraction*D/2 (highest frequencies)."""
    return int(round(fraction * head_dim / 2))


def rope_cos_sin(pos, head_dim: int, theta: float, fraction: float):
    """cos/sin of position * theta_i for the rotated pairs, rounded to binary32.

    Angles and trigonometry are float64; the kernels hold the factors in
    binary32, so they are rounded to it here.  Returns two [npos, n_rot]
    float32 arrays."""
    n = rope_rotated_pairs(head_dim, fraction)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(head_dim, theta)[None, :n]
    return f32(np.cos(ang)), f32(np.sin(ang))


def rope(x, pos, head_dim: int, theta: float, fraction: float) -> np.ndarray:
    """Rotate-half RoPE applied to the first fraction*D/2 pairs.

    x: [npos, H, D] binary32 values; pos: [npos].  Pair i couples dimension
    i with i + D/2: (a, b) -> (a*c - b*s, a*s + b*c).  The arithmetic is
    binary32 with every product and sum rounded on its own (no fused
    multiply-add), the precision in which the bf16 value stored afterwards
    is decided.  Unrotated pairs pass through unchanged."""
    x = np.array(x, dtype=np.float32, copy=True)
    n = rope_rotated_pairs(head_dim, fraction)
    if n == 0:
        return x
    c, s = rope_cos_sin(pos, head_dim, theta, fraction)
    c = c[:, None, :]
    s = s[:, None, :]
    h = head_dim // 2
    a = x[..., :n].copy()
    b = x[..., h:h + n].copy()
    x[..., :n] = (a * c) - (b * s)
    x[..., h:h + n] = (a * s) + (b * c)
    return x


# ---------------------------------------------------------------------------
# Attention, LM head, acceptance
# ---------------------------------------------------------------------------


def attend(q, keys, vals, qpos, kpos, window: int, scale: float) -> np.ndarray:
    """Softmax attention of query rows over keys, computed directly.

    q [R][D], keys/vals [J][D] (any float), qpos [R], kpos [J].  Key j is
    visible to row r iff kpos[j] <= qpos[r] and, for window > 0,
    kpos[j] > qpos[r] - window.  All visible scores q.k*scale are formed,
    the row maximum subtracted, exponentiated, normalised, and the values
    summed with those weights (float64).  Returns [R][D] float64."""
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    vals = np.asarray(vals, dtype=np.float64)
    qpos = np.asarray(qpos, dtype=np.int64)
    kpos = np.asarray(kpos, dtype=np.int64)
    s = (q @ keys.T) * scale
    vis = kpos[None, :] <= qpos[:, None]
    if window > 0:
        vis &= kpos[None, :] > qpos[:, None] - window
    if not np.all(vis.any(axis=1)):
        raise ValueError("a query row sees no key")
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.where(vis, np.exp(s - m), 0.0)
    return (p @ vals) / p.sum(axis=1, keepdims=True)


def lm_head_top2(h, w_bits, chunk: int = 8192):
    """Logits h . W_v over the vocabulary, argmax and runner-up.

    h [M][d] (float), w_bits [V][d] bf16 bit patterns.  Each logit is a
    float64 dot product rounded to binary32 (the format the argmax is
    decided in); the argmax is the first maximum (lowest token id on ties).
    Returns (ids int64 [M], top1 float64 [M], top2 float64 [M])."""
    h = np.asarray(h, dtype=np.float64)
    M = h.shape[0]
    V = w_bits.shape[0]
    ids = np.zeros(M, dtype=np.int64)
    top1 = np.full(M, -np.inf)
    top2 = np.full(M, -np.inf)
    rows = np.arange(M)
    for v0 in range(0, V, chunk):
        wc = bf16_from_bits(w_bits[v0:v0 + chunk]).astype(np.float64)
        lg = f32(h @ wc.T).astype(np.float64)            # [M][chunk]
        j = np.argmax(lg, axis=1)                        # first maximum in the chunk
        c1 = lg[rows, j]
        lg2 = lg.copy()
        lg2[rows, j] = -np.inf
        c2 = lg2.max(axis=1) if lg2.shape[1] > 1 else np.full(M, -np.inf)
        better = c1 > top1                               # strict: earlier chunk wins ties
        new_top2 = np.where(better, np.maximum(top1, c2), np.maximum(top2, c1))
        top1 = np.where(better, c1, top1)
        ids = np.where(better, v0 + j, ids)
        top2 = new_top2
    return ids, top1, top2


def accept_longest_prefix(drafts, g):
    """Longest matching prefix plus the target's own token ([P1] §4.1/§4.2,
    [P2] §3, [P3] §什么是多标记预测).

    drafts [k], g [k+1] (the target's argmax at rows 0..k).  a is the number
    of leading drafts equal to the target's choice; the step emits those a
    drafts followed by g[a] (when all k agree, g[k] is the extra token).
    Returns (a, emitted [k+1] with -1 padding, next last token g[a])."""
    drafts = [int(t) for t in drafts]
    g = [int(t) for t in g]
    k = len(drafts)
    a = 0
    while a < k and drafts[a] == g[a]:
        a += 1
    emitted = drafts[:a] + [g[a]] + [-1] * (k - a)
    return a, emitted, g[a]


# ---------------------------------------------------------------------------
# The synthetic target model and its cache
# ---------------------------------------------------------------------------


@dataclass
class LayerDef:
    window: int                  # 0 = global
    kv_equal: bool               # V is the pre-RoPE key
    rope_fraction: float
    w_qkv: np.ndarray            # float32 values [Nqkv][d]: rows q heads | k heads | v heads
    w_o: np.ndarray              # float32 values [d][Hq*D]


@dataclass
class Model:
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    w_lm_bits: np.ndarray        # [V][d] bf16 bits: LM head
    layers: list
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    w_emb_bits: np.ndarray | None = None   # [V][d] token embedding; None: tied to the LM head

    @property
    def vocab(self) -> int:
        return self.w_lm_bits.shape[0]


@dataclass
class LayerCache:
    """Cache of one layer for one sequence, positions [lo, lo + n).

    k: post-RoPE keys; v: values (separate-K/V layers) or None; kpre: the
    pre-RoPE keys, which are the values on key-equals-value layers."""
    lo: int
    k: np.ndarray                # float32 [n][Hkv][D]
    v: np.ndarray | None
    kpre: np.ndarray | None

    @property
    def end(self) -> int:
        return self.lo + self.k.shape[0]

    def values(self) -> np.ndarray:
        return self.kpre if self.v is None else self.v


def kv_values_per_token_head(head_dim: int, fraction: float, kv_equal: bool) -> int:
    """Values a layer must keep per cached token and KV head.

    Separate K/V: D keys + D values.  Key-equals-value: the D post-RoPE keys
    plus the pre-RoPE values of the 2*p*D/2 rotated dimensions (the only
    ones RoPE changed), from which V = pre-RoPE K is recovered without
    arithmetic ([P1] §2: the global cache shrinks by 37.5% at p = 0.25)."""
    if not kv_equal:
        return 2 * head_dim
    return head_dim + 2 * rope_rotated_pairs(head_dim, fraction)


def cache_from_raw(model: Model, l: int, lo: int, k_raw, v_raw) -> LayerCache:
    """Cache entries for context positions lo.. from raw pre-RoPE keys/values.

    k_raw/v_raw: float32 values of bf16 draws [n][Hkv][D]; v_raw is None on
    key-equals-value layers."""
    spec = model.layers[l]
    k_raw = np.asarray(k_raw, dtype=np.float32)
    pos = np.arange(lo, lo + k_raw.shape[0])
    k = bf16(rope(k_raw, pos, model.head_dim, model.rope_theta, spec.rope_fraction))
    if spec.kv_equal:
        return LayerCache(lo, k, None, bf16(k_raw))
    return LayerCache(lo, k, bf16(v_raw), None)


def attention_layer(model: Model, l: int, cache: LayerCache, L: int, q_pre, k_pre, v_pre):
    """One layer's verify attention for one sequence.

    q_pre [q][Hq][D], k_pre [q][Hkv][D], v_pre [q][Hkv][D] or None: the
    projections of the q rows (positions L..L+q-1) before RoPE, binary32
    values.  The rows' keys are rotated, rounded to bf16 and appended after
    the cache's positions; each query head h reads KV head h // (Hq/Hkv)
    (grouped-query attention) with the causal + window mask of `attend`.

    Returns (out bf16-valued [q][Hq][D], new entries (k, v, kpre) for
    positions L..L+q-1)."""
    spec = model.layers[l]
    D, Hq, Hkv = model.head_dim, model.n_q_heads, model.n_kv_heads
    if cache.end != L:
        raise ValueError("cache does not end at the committed length")
    nq = q_pre.shape[0]
    pos = np.arange(L, L + nq)
    q_rot = bf16(rope(q_pre, pos, D, model.rope_theta, spec.rope_fraction))
    k_new = bf16(rope(k_pre, pos, D, model.rope_theta, spec.rope_fraction))
    if spec.kv_equal:
        v_new, kpre_new = None, bf16(k_pre)
        vals_new = kpre_new
    else:
        v_new, kpre_new = bf16(v_pre), None
        vals_new = v_new
    keys = np.concatenate([cache.k, k_new], axis=0)
    vals = np.concatenate([cache.values(), vals_new], axis=0)
    kpos = np.arange(cache.lo, L + nq)
    G = Hq // Hkv
    out = np.empty((nq, Hq, D), dtype=np.float64)
    scale = 1.0 / np.sqrt(D)
    for h in range(Hq):
        kh = h // G
        out[:, h, :] = attend(q_rot[:, h, :], keys[:, kh, :], vals[:, kh, :], pos, kpos,
                              spec.window, scale)
    return bf16(out), (k_new, v_new, kpre_new)


@dataclass
class Forward:
    g: np.ndarray                # argmax token of each LM-head row
    top1: np.ndarray
    top2: np.ndarray
    h: np.ndarray                # final hidden state (bf16 values) of the LM-head rows
    new_entries: list            # per layer (k, v, kpre) for positions L..L+q-1
    attn_out: list               # per layer bf16 attention output [q][Hq][D]
    x_out: np.ndarray            # residual stream after the last layer (binary32)


def verify_forward(model: Model, caches: list, L: int, tokens, lm_rows=None) -> Forward:
    """The target's one-forward verification of q = len(tokens) rows ([P1] §4.2
    `main_model.verify`; [P2] §3).

    tokens [q] = [last accepted token, drafts...] at positions L..L+q-1.
    caches[l] holds positions up to L-1.  lm_rows selects the rows whose
    logits are formed (default all)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    nq = tokens.shape[0]
    D, Hq, Hkv = model.head_dim, model.n_q_heads, model.n_kv_heads
    emb = model.w_lm_bits if model.w_emb_bits is None else model.w_emb_bits
    x = bf16_from_bits(emb[tokens]).astype(np.float32)                   # embedding rows
    new_entries, attn_out = [], []
    for l, spec in enumerate(model.layers):
        hn = bf16(rmsnorm(x, model.rms_eps))
        qkv = f32(hn.astype(np.float64) @ spec.w_qkv.astype(np.float64).T)
        q_pre = qkv[:, :Hq * D].reshape(nq, Hq, D)
        k_pre = qkv[:, Hq * D:(Hq + Hkv) * D].reshape(nq, Hkv, D)
        v_pre = None if spec.kv_equal else qkv[:, (Hq + Hkv) * D:].reshape(nq, Hkv, D)
        o, ent = attention_layer(model, l, caches[l], L, q_pre, k_pre, v_pre)
        new_entries.append(ent)
        attn_out.append(o)
        y = f32(o.reshape(nq, Hq * D).astype(np.float64) @ spec.w_o.astype(np.float64).T)
        x = f32(x.astype(np.float64) + y.astype(np.float64))
    rows = np.arange(nq) if lm_rows is None else np.asarray(lm_rows, dtype=np.int64)
    h = bf16(rmsnorm(x[rows], model.rms_eps))
    if rows.size == 0:                      # caller forms the logits itself (batched)
        empty = np.zeros(0)
        return Forward(empty.astype(np.int64), empty, empty, h, new_entries, attn_out, x)
    g, t1, t2 = lm_head_top2(h, model.w_lm_bits)
    return Forward(g, t1, t2, h, new_entries, attn_out, x)


def commit(caches: list, fw: Forward, n_rows: int) -> list:
    """Caches extended by the first n_rows new entries of a forward (the
    accepted rows); the other rows are rolled back, i.e. never appended."""
    out = []
    for c, (k, v, kp) in zip(caches, fw.new_entries):
        out.append(LayerCache(
            c.lo,
            np.concatenate([c.k, k[:n_rows]], axis=0),
            None if v is None else np.concatenate([c.v, v[:n_rows]], axis=0),
            None if kp is None else np.concatenate([c.kpre, kp[:n_rows]], axis=0),
        ))
    return out


@dataclass
class StepResult:
    g: np.ndarray
    top1: np.ndarray
    top2: np.ndarray
    accept_len: int
    emitted: list
    next_last_token: int
    new_len: int
    forward: Forward


def verify_step(model: Model, caches: list, L: int, last_token: int, drafts) -> StepResult:
    """One verify step: forward over [last_token, drafts], accept the longest
    matching prefix, add the target's token, commit a+1 positions
    ([P1] §4.2 `speculative_step` steps 2-3)."""
    drafts = [int(t) for t in drafts]
    fw = verify_forward(model, caches, L, [int(last_token)] + drafts)
    a, emitted, nxt = accept_longest_prefix(drafts, fw.g)
    return StepResult(fw.g, fw.top1, fw.top2, a, emitted, nxt, L + a + 1, fw)


def prefill(model: Model, tokens, chunk: int | None = None) -> tuple:
    """Cache of a prompt: forward over the prompt tokens from an empty cache
    (positions 0..n-1), committing every row.  Returns (caches, g of the
    last row, top1, top2)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    D, Hkv = model.head_dim, model.n_kv_heads
    empty = np.zeros((0, Hkv, D), dtype=np.float32)
    caches = [LayerCache(0, empty, None if s.kv_equal else empty, empty if s.kv_equal else None)
              for s in model.layers]
    n = tokens.shape[0]
    step = n if chunk is None else chunk
    L = 0
    fw = None
    while L < n:
        part = tokens[L:L + step]
        fw = verify_forward(model, caches, L, part, lm_rows=[part.shape[0] - 1])
        caches = commit(caches, fw, part.shape[0])
        L += part.shape[0]
    return caches, int(fw.g[0]), float(fw.top1[0]), float(fw.top2[0])


def greedy_decode(model: Model, caches: list, L: int, last_token: int, n_tokens: int):
    """Plain token-by-token greedy decoding: one forward per token.
    Returns (tokens emitted, top1-top2 margins, caches, final length)."""
    out, margins = [], []
    tok = int(last_token)
    for _ in range(n_tokens):
        fw = verify_forward(model, caches, L, [tok])
        caches = commit(caches, fw, 1)
        L += 1
        tok = int(fw.g[0])
        out.append(tok)
        margins.append(float(fw.top1[0] - fw.top2[0]))
    return out, margins, caches, L


def speculative_decode(model: Model, caches: list, L: int, last_token: int, k: int,
                       n_tokens: int, drafter):
    """Speculative loop ([P1] §4.2 `speculative_step`): at each step
    drafter(step, emitted_so_far, k) proposes k tokens, the target verifies
    them, the accepted prefix plus the target's token are emitted and
    committed.  Stops once n_tokens are emitted (the last step may overshoot;
    the stream is cut to n_tokens).  Returns (tokens, accept lengths)."""
    out, accepts = [], []
    tok = int(last_token)
    step = 0
    while len(out) < n_tokens:
        drafts = drafter(step, list(out), k)
        res = verify_step(model, caches, L, tok, drafts)
        caches = commit(caches, res.forward, res.accept_len + 1)
        L = res.new_len
        out.extend(res.emitted[:res.accept_len + 1])
        accepts.append(res.accept_len)
        tok = res.next_last_token
        step += 1
    return out[:n_tokens], accepts
