"""The synthetic verify-step workloads and their seeded raw inputs.

Shapes follow the five benchmark configurations (tiny one-layer step; batch 1
at 8k context with a sliding-window and a key-equals-value global layer;
batch 8 ragged 4k-32k global-only; batch 64 six-layer throughput case; the
4-layer 131k-prompt speculative loop), plus scaled-down variants of the same
structure for parity tests that the CPU oracle finishes in seconds.

Everything here is a draw or a layout decision: weights N(0, 0.02) bf16,
context pre-RoPE keys/values N(0, 1) bf16, token ids uniform, the per-token
accept coin flips that decide where a draft first goes wrong, and a seeded
random permutation of the page pool.  No model arithmetic happens here.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np

from . import gen

PAGE = 64


@dataclass(frozen=True)
class LayerSpec:
    window: int = 0            # 0 = global attention; else sliding window (keys incl. self)
    kv_equal: bool = False     # key-equals-value global layer (V = pre-RoPE K)
    rope_fraction: float = 1.0 # fraction of rotary pairs rotated (highest frequencies first)
    split_tokens: int = 0      # split-KV chunk of this layer (0: the workload's)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    k: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    vocab: int
    layers: tuple
    ctx_lo: int                 # context lengths uniform in [ctx_lo, ctx_hi] (inclusive)
    ctx_hi: int
    accept: tuple               # draft recipe, see make_drafts
    split_tokens: int = 256     # absolute split-KV chunk of the attention reduction
    page_size: int = PAGE
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    weight_std: float = 0.02
    seed: int = 0
    steps: int = 1              # verify steps (the loop workload runs many)
    prompt_tokens: int = 0      # >0: context is a prefilled random prompt, not drawn K/V
    tied_embedding: bool = False

    @property
    def q_rows(self) -> int:
        return self.k + 1

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def qkv_out(self, layer: LayerSpec) -> int:
        nv = 0 if layer.kv_equal else self.n_kv_heads
        return (self.n_q_heads + self.n_kv_heads + nv) * self.head_dim

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


LOCAL1024 = LayerSpec(window=1024, kv_equal=False, rope_fraction=1.0, split_tokens=128)
GLOBAL_KV = LayerSpec(window=0, kv_equal=True, rope_fraction=0.25)
GLOBAL_FULL = LayerSpec(window=0, kv_equal=False, rope_fraction=1.0)

WORKLOADS = {
    # Tiny verify step: 1 layer, 8 q heads / 1 kv head, D 128, d 512, V 4096, ctx 256.
    "tiny": Workload("tiny", batch=1, k=4, d_model=512, n_q_heads=8, n_kv_heads=1, head_dim=128,
                     vocab=4096, layers=(GLOBAL_FULL,), ctx_lo=256, ctx_hi=256,
                     accept=("one_wrong", 0.5)),
    # Batch 1, 8k context, k=4: sliding-window layer + key-equals-value global layer.
    "b1_ctx8k": Workload("b1_ctx8k", batch=1, k=4, d_model=2560, n_q_heads=16, n_kv_heads=8,
                         head_dim=256, vocab=262144, layers=(LOCAL1024, GLOBAL_KV),
                         ctx_lo=8192, ctx_hi=8192, accept=("geometric", 0.8), split_tokens=256),
    # Batch 8 ragged 4k-32k, global key-equals-value layer only.
    "b8_ragged": Workload("b8_ragged", batch=8, k=4, d_model=5376, n_q_heads=32, n_kv_heads=4,
                          head_dim=256, vocab=262144, layers=(GLOBAL_KV,), ctx_lo=4096,
                          ctx_hi=32768, accept=("geometric", 0.8), split_tokens=1024),
    # Batch 64, k=3, 5 sliding-window layers + 1 key-equals-value global layer.
    # (64 sequences x 8 KV heads already fill the GPU: long splits keep the
    #  split-combine traffic small)
    "b64_6layer": Workload("b64_6layer", batch=64, k=3, d_model=3840, n_q_heads=16, n_kv_heads=8,
                           head_dim=256, vocab=262144,
                           layers=(LOCAL1024.__class__(window=1024, split_tokens=1024),) * 5
                           + (GLOBAL_KV,), ctx_lo=1024, ctx_hi=16384,
                           accept=("geometric_per_seq", 0.5, 0.9), split_tokens=2048),
    # Speculative loop: 4 layers (3 sliding + 1 global K=V), 131072-token prompt, k=8, 512 steps.
    "loop_131k": Workload("loop_131k", batch=1, k=8, d_model=2048, n_q_heads=8, n_kv_heads=2,
                          head_dim=256, vocab=262144, layers=(LOCAL1024,) * 3 + (GLOBAL_KV,),
                          ctx_lo=131072, ctx_hi=131072, accept=("corrupted_greedy", 0.8),
                          split_tokens=1024, steps=512, prompt_tokens=131072),
}

# Scaled-down variants with the same structure, sized for the CPU oracle to
# finish in seconds while still spanning several tiles, pages and splits and
# leaving ragged tails (vocab not a multiple of the 128-row tile, contexts
# not a multiple of the 64-token page or the split).
WORKLOADS.update({
    "small_b1": WORKLOADS["b1_ctx8k"].with_(name="small_b1", vocab=9000, ctx_lo=1500, ctx_hi=1500,
                                              layers=(LayerSpec(window=300, split_tokens=128),
                                                      GLOBAL_KV)),
    "small_ragged": WORKLOADS["b8_ragged"].with_(name="small_ragged", batch=4, d_model=1024,
                                                  vocab=5000, ctx_lo=100, ctx_hi=1400),
    "small_b16": WORKLOADS["b64_6layer"].with_(name="small_b16", batch=16, d_model=768,
                                                vocab=4100, ctx_lo=60, ctx_hi=900,
                                                layers=(LayerSpec(window=200, split_tokens=64),) * 2
                                                + (GLOBAL_KV,)),
    # 32 sequences x 4 rows = 128 verify rows: the many-row (tensor-memory) GEMM path
    "small_b32": WORKLOADS["b64_6layer"].with_(name="small_b32", batch=32, d_model=768,
                                                vocab=4100, ctx_lo=60, ctx_hi=700,
                                                layers=(LayerSpec(window=200, split_tokens=64),
                                                        GLOBAL_KV)),
    # the window of the first verify row starts on the last key of a split
    # (1450 - 300 + 1 = 9 * 128 - 1), so each later row's window starts in the
    # next split: the split combine must not depend on where the list begins
    "small_b1_edge": WORKLOADS["b1_ctx8k"].with_(name="small_b1_edge", vocab=9000, ctx_lo=1450,
                                                   ctx_hi=1450,
                                                   layers=(LayerSpec(window=300, split_tokens=128),
                                                           GLOBAL_KV)),
    # the largest draft count the library takes: 17 verify rows
    "small_b1_k16": WORKLOADS["b1_ctx8k"].with_(name="small_b1_k16", k=16, vocab=9000, ctx_lo=1500,
                                                  ctx_hi=1500,
                                                  layers=(LayerSpec(window=300, split_tokens=128),
                                                          GLOBAL_KV)),
    # 40 sequences x 9 rows = 360 verify rows: more rows than one tensor-memory
    # accumulator holds (256), so every GEMM takes the multi-block path
    "small_b40_k8": WORKLOADS["b64_6layer"].with_(name="small_b40_k8", batch=40, k=8, d_model=768,
                                                   vocab=5000, ctx_lo=60, ctx_hi=500,
                                                   accept=("geometric", 0.8),
                                                   layers=(LayerSpec(window=200, split_tokens=64),
                                                           GLOBAL_KV)),
    "small_loop": WORKLOADS["loop_131k"].with_(name="small_loop", vocab=6000, d_model=512,
                                                ctx_lo=700, ctx_hi=700, prompt_tokens=700,
                                                layers=(LayerSpec(window=128),) * 3 + (GLOBAL_KV,),
                                                split_tokens=256, steps=24),
})


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


# --------------------------------------------------------------------------
# Weights
# --------------------------------------------------------------------------

def _w(wl: Workload, name: str, rows: int, cols: int) -> np.ndarray:
    out = gen.normal_bf16(wl.seed, f"{wl.name}/{name}", 0, rows * cols, wl.weight_std)
    return out.reshape(rows, cols)


def lm_head_weight(wl: Workload) -> np.ndarray:
    """LM-head matrix, bf16 bits, [vocab][d_model]."""
    return _w(wl, "w_lm", wl.vocab, wl.d_model)


def embedding_weight(wl: Workload):
    """Token embedding, bf16 bits, [vocab][d_model]; None when tied to the LM head.

    Untied by default: with random weights a tied table makes every token's
    own logit dominate (the model copies its input), which would leave the
    acceptance path untested by the model's choices."""
    if wl.tied_embedding:
        return None
    return _w(wl, "w_emb", wl.vocab, wl.d_model)


DRAFT_WIDTH = 256       # drafter block width of the small models' drafters
DRAFT_BLOCKS = 4        # three sliding-window blocks, then one global block


def drafter_spec(wl: Workload):
    """(d_draft, n_q_heads, target layer of each block): the sliding-window
    blocks read the target's last sliding-window layer, the global block its
    last global layer (either kind stands in when the target lacks the
    other)."""
    local = [l for l, s in enumerate(wl.layers) if s.window > 0]
    glob = [l for l, s in enumerate(wl.layers) if s.window == 0]
    last_local = local[-1] if local else glob[-1]
    last_global = glob[-1] if glob else local[-1]
    targets = [last_local] * (DRAFT_BLOCKS - 1) + [last_global]
    return min(DRAFT_WIDTH, wl.d_model), wl.n_q_heads, targets


def drafter_weights(wl: Workload):
    """Drafter weights, bf16 bits: (embedding [vocab][d_draft], W_down
    [d_draft][d_model + d_draft], W_up [d_model][d_draft], blocks [(W_q
    [Hq*D][d_draft], W_o [d_draft][Hq*D], target layer)])."""
    dd, hq, targets = drafter_spec(wl)
    nq = hq * wl.head_dim
    emb = _w(wl, "draft/w_emb", wl.vocab, dd)
    down = _w(wl, "draft/w_down", dd, wl.d_model + dd)
    upw = _w(wl, "draft/w_up", wl.d_model, dd)
    blocks = [(_w(wl, f"draft/b{i}/w_q", nq, dd), _w(wl, f"draft/b{i}/w_o", dd, nq), t)
              for i, t in enumerate(targets)]
    return emb, down, upw, blocks


def drafter_inputs(wl: Workload, b: int, attempt: int):
    """(target activation bf16 bits [d_model], previous token) of sequence b."""
    key = f"{wl.name}/draft_in/b{b}/a{attempt}"
    return (gen.normal_bf16(wl.seed, key + "/h", 0, wl.d_model, 1.0),
            int(gen.randint(wl.seed, key + "/tok", 0, 1, 0, wl.vocab)[0]))


CLUSTER_SIZE = 128      # tokens per cluster of the cheap unembedding
CANDIDATES = 4096       # candidate tokens per row it aims for (~4096)


def _permutation(wl: Workload, name: str, n: int) -> np.ndarray:
    u = gen.uniform(wl.seed, f"{wl.name}/{name}", 0, n)
    perm = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):           # Fisher-Yates, driven by the counter stream
        j = int(u[i] * (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bf16 bit patterns, round to nearest even (storage format only)."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


def cluster_tables(wl: Workload, w_lm_bits=None):
    """Synthetic token clusters for the cheap unembedding: a seeded random
    partition of the vocabulary into clusters of CLUSTER_SIZE tokens (the
    last one padded with -1), each cluster's centroid the mean of its
    members' LM-head rows (bf16), and the LM-head rows copied in cluster
    order (zero rows for the padding).  Returns (cluster_tokens [C][S]
    int32, centroid bits [C][d], clustered LM-head bits [C*S][d],
    n_select)."""
    S, V, d = CLUSTER_SIZE, wl.vocab, wl.d_model
    C = -(-V // S)
    perm = _permutation(wl, "clusters", V)
    toks = np.full(C * S, -1, dtype=np.int32)
    toks[:V] = perm
    w = lm_head_weight(wl) if w_lm_bits is None else w_lm_bits
    wc = np.zeros((C * S, d), dtype=np.uint16)
    wc[:V] = w[perm]
    vals = (wc.astype(np.uint32) << 16).view(np.float32).reshape(C, S, d)
    counts = (toks.reshape(C, S) >= 0).sum(axis=1)
    cent = _bf16_bits(vals.astype(np.float64).sum(axis=1) / counts[:, None])
    n_select = min(CANDIDATES // S, max(1, C // 8))
    return toks.reshape(C, S), cent, wc, n_select


def layer_weights(wl: Workload, l: int):
    """(W_qkv [Nqkv][d], W_o [d][Hq*D]) bf16 bits, rows = output features.

    W_qkv rows are ordered [q heads | k heads | v heads (absent on K=V layers)],
    each head's head_dim rows contiguous."""
    spec = wl.layers[l]
    wqkv = _w(wl, f"l{l}/w_qkv", wl.qkv_out(spec), wl.d_model)
    wo = _w(wl, f"l{l}/w_o", wl.d_model, wl.n_q_heads * wl.head_dim)
    return wqkv, wo


# --------------------------------------------------------------------------
# Per-sequence inputs
# --------------------------------------------------------------------------

def context_lengths(wl: Workload) -> np.ndarray:
    if wl.ctx_lo == wl.ctx_hi:
        return np.full(wl.batch, wl.ctx_lo, dtype=np.int64)
    return gen.randint(wl.seed, f"{wl.name}/ctx_len", 0, wl.batch, wl.ctx_lo, wl.ctx_hi + 1)


def visible_start(wl: Workload, spec: LayerSpec, L: int) -> int:
    """First context position any of the q rows (positions L..L+k) can see.

    Row at position t sees keys j with t - W < j <= t on a window-W layer, so
    over the rows the earliest visible key is L - W + 1."""
    if spec.window == 0:
        return 0
    return max(0, L - spec.window + 1)


def context_kv(wl: Workload, b: int, attempt: int, l: int, L: int):
    """Raw (pre-RoPE) context keys and values for positions [lo, L) of layer l.

    Returns (lo, k_raw [n][Hkv][D] bf16 bits, v_raw or None).  Element
    (pos j, head h, dim e) is counter (j*Hkv + h)*D + e of its stream, so a
    position's values do not depend on which slice is generated.  K=V layers
    have no separate V."""
    spec = wl.layers[l]
    lo = visible_start(wl, spec, L)
    n = L - lo
    hd = wl.n_kv_heads * wl.head_dim
    base = f"{wl.name}/b{b}/t{attempt}/l{l}"
    k = gen.normal_bf16(wl.seed, base + "/ctx_k", lo * hd, n * hd, 1.0).reshape(n, wl.n_kv_heads,
                                                                                 wl.head_dim)
    v = None
    if not spec.kv_equal:
        v = gen.normal_bf16(wl.seed, base + "/ctx_v", lo * hd, n * hd, 1.0).reshape(
            n, wl.n_kv_heads, wl.head_dim)
    return lo, k, v


def last_token(wl: Workload, b: int, attempt: int) -> int:
    return int(gen.randint(wl.seed, f"{wl.name}/b{b}/t{attempt}/last_token", 0, 1, 0, wl.vocab)[0])


def prompt_tokens(wl: Workload, b: int = 0) -> np.ndarray:
    """Random prompt token ids for the prefilled-loop workload."""
    return gen.randint(wl.seed, f"{wl.name}/b{b}/prompt", 0, wl.prompt_tokens, 0, wl.vocab)


def rejection_point(wl: Workload, b: int, attempt: int) -> int:
    """Index r of the first wrong draft (r == k: all drafts correct).

    geometric(p): r = number of leading successes of per-token Bernoulli(p)
    coin flips, capped at k.  geometric_per_seq(lo, hi): the same with
    p_b ~ U[lo, hi] drawn once per sequence.  one_wrong(q): with probability
    q one position j ~ U[0, k) is wrong, else none."""
    kind = wl.accept[0]
    base = f"{wl.name}/b{b}/t{attempt}"
    if kind == "one_wrong":
        coin = gen.uniform(wl.seed, base + "/wrong_coin", 0, 1)[0]
        if coin < wl.accept[1]:
            return int(gen.randint(wl.seed, base + "/wrong_pos", 0, 1, 0, wl.k)[0])
        return wl.k
    if kind == "geometric":
        p = wl.accept[1]
    elif kind == "geometric_per_seq":
        p = wl.accept[1] + (wl.accept[2] - wl.accept[1]) * gen.uniform(
            wl.seed, f"{wl.name}/b{b}/accept_p", 0, 1)[0]
    else:
        raise ValueError(f"no fixed rejection point for draft recipe {kind}")
    flips = gen.uniform(wl.seed, base + "/accept_flips", 0, wl.k)
    r = 0
    while r < wl.k and flips[r] < p:
        r += 1
    return r


def make_drafts(wl: Workload, b: int, attempt: int, greedy: np.ndarray,
                r: int | None = None) -> tuple[np.ndarray, int]:
    """Drafts from the greedy continuation `greedy` (at least r+1 tokens).

    drafts[i] = greedy[i] for i < r; drafts[r] = a random id != greedy[r];
    later drafts are random ids.  one_wrong keeps greedy tokens after the
    replaced position.  r defaults to rejection_point(wl, b, attempt); a
    caller that keeps a sequence's rejection point fixed across redraws of
    its context passes it.  Returns (drafts[k] int32, r)."""
    if r is None:
        r = rejection_point(wl, b, attempt)
    stream = f"{wl.name}/b{b}/t{attempt}/draft_rand"
    ids = gen.randint(wl.seed, stream, 0, 4 * wl.k + 64, 0, wl.vocab)
    drafts = np.empty(wl.k, dtype=np.int32)
    ctr = 0
    for i in range(wl.k):
        if i < r:
            drafts[i] = greedy[i]
        elif i == r:
            while ids[ctr] == greedy[r]:
                ctr += 1
            drafts[i] = ids[ctr]
            ctr += 1
        elif wl.accept[0] == "one_wrong":
            drafts[i] = greedy[i]
        else:
            drafts[i] = ids[ctr]
            ctr += 1
    return drafts, r


def loop_draft_flips(wl: Workload, step: int) -> tuple[np.ndarray, np.ndarray]:
    """Coin flips and random ids of the corrupted-greedy drafter at one loop step:
    draft i is the true greedy token if flip[i] < p else ids[i]."""
    flips = gen.uniform(wl.seed, f"{wl.name}/loop_flips", step * wl.k, wl.k)
    ids = gen.randint(wl.seed, f"{wl.name}/loop_ids", step * wl.k, wl.k, 0, wl.vocab)
    return flips, ids


# --------------------------------------------------------------------------
# Paged layout
# --------------------------------------------------------------------------

def pages_needed(L: int, k: int, page: int = PAGE, extra_tokens: int = 0) -> int:
    return -(-(L + k + 1 + extra_tokens) // page)


def page_assignment(wl: Workload, lens, extra_tokens: int = 0):
    """Seeded random permutation of the pool, handed out sequence by sequence.

    Returns (num_pages, block_table [B][max_pages] int32, -1 padded)."""
    need = [pages_needed(int(L), wl.k, wl.page_size, extra_tokens) for L in lens]
    total = int(sum(need))
    u = gen.uniform(wl.seed, f"{wl.name}/page_perm", 0, total)
    perm = np.arange(total, dtype=np.int64)
    for i in range(total - 1, 0, -1):       # Fisher-Yates, driven by the counter stream
        j = int(u[i] * (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    maxp = max(need)
    table = np.full((len(lens), maxp), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[pos:pos + n]
        pos += n
    return total, table
