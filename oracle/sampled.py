"""Oracle of distribution-preserving (sampled) verification.

TEST INFRASTRUCTURE ONLY (see the package docstring).  float64 arithmetic on
binary32 logits.

The pages state the property only: [P3] "Gemma 4 发布时未包含 MTP 数据——为什么这很重要"
§MTP 能快多少 says the output is identical to what standard decoding produces,
and [P1] §4.1 / [P2] §3 describe the target checking the drafts in one
forward and keeping the agreeing run.  For sampling (rather than greedy)
decoding the standard way to keep that property is speculative sampling
(Leviathan, Kalman, Matias, "Fast Inference from Transformers via
Speculative Decoding", ICML 2023, Algorithm 1; Chen et al., "Accelerating
Large Language Model Decoding with Speculative Sampling", 2023), which this
follows:

  for i = 0..k-1: accept draft d_i iff u_i < p_i(d_i) / q_i(d_i) (always when
  p_i(d_i) >= q_i(d_i)); at the first rejection emit a token drawn from
  norm(max(0, p_i - q_i)) and stop; if every draft is accepted, emit a token
  drawn from p_k.  The emitted sequence is then distributed exactly as
  sampling from the target alone.

Readings where the method leaves a step open:
  * p_i = softmax(target logits of verify row i / T), q_i = softmax(draft
    logits of draft step i / T), T the sampling temperature (T > 0);
  * the acceptance test is u_i * q_i(d_i) < p_i(d_i) with u_i uniform in
    [0, 1) (no division);
  * a draw from weights w over the vocabulary is the Gumbel-max choice
    argmax_v (log w_v - log(-log g_v)) with g_v uniform in (0, 1); tokens
    with w_v = 0 are never drawn; equal scores go to the lowest token id;
  * the random numbers are inputs: u [k] per sequence and g [V] for the one
    draw a sequence makes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .verify import bf16_from_bits, f32

__all__ = ["softmax", "gumbel_draw", "SampledResult", "speculative_sample", "full_logits"]


def full_logits(h, w_bits, chunk: int = 16384) -> np.ndarray:
    """Logits h . W_v of every token (float64 products rounded to binary32),
    the LM head's definition: h [M][d] bf16 values, w_bits [V][d] bf16 bits."""
    h = np.asarray(h, dtype=np.float64)
    out = np.empty((h.shape[0], w_bits.shape[0]), dtype=np.float32)
    for v0 in range(0, w_bits.shape[0], chunk):
        out[:, v0:v0 + chunk] = f32(h @ bf16_from_bits(w_bits[v0:v0 + chunk]).astype(np.float64).T)
    return out


def softmax(logits, T: float = 1.0) -> np.ndarray:
    """softmax(logits / T) over the last axis, float64."""
    z = np.asarray(logits, dtype=np.float64) / T
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def gumbel_draw(w, g):
    """Token drawn from weights w >= 0 with uniforms g: argmax_v log w_v -
    log(-log g_v) (w_v = 0 excluded; ties: lowest id).  Returns (token, best
    score, second score, second token)."""
    w = np.asarray(w, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(divide="ignore"):
        score = np.where(w > 0, np.log(w) - np.log(-np.log(g)), -np.inf)
    j = int(np.argmax(score))
    rest = score.copy()
    rest[j] = -np.inf
    j2 = int(np.argmax(rest))
    return j, float(score[j]), float(rest[j2]), j2


@dataclass
class SampledResult:
    accept_len: int
    emitted: list                # accepted drafts, then the drawn token; -1 padding to k+1
    next_last_token: int
    accept_margin: float         # min over tested drafts of |u q - p| / max(u q, p)
    draw_margin: float           # best minus second Gumbel score of the draw
    draw_weights: tuple          # ((p, q) of the drawn token, (p, q) of the runner-up); q = 0 for p_k


def speculative_sample(p_logits, q_logits, drafts, u, g, T: float = 1.0) -> SampledResult:
    """Speculative sampling of one sequence.

    p_logits [k+1][V]: target logits of verify rows 0..k (binary32);
    q_logits [k][V]: draft logits of draft steps 0..k-1; drafts [k];
    u [k] acceptance uniforms; g [V] draw uniforms."""
    drafts = [int(d) for d in drafts]
    k = len(drafts)
    p = softmax(p_logits, T)
    q = softmax(q_logits, T) if k else np.zeros((0, p.shape[1]))
    margin = np.inf
    a = 0
    while a < k:
        pd, qd = p[a, drafts[a]], q[a, drafts[a]]
        margin = min(margin, abs(u[a] * qd - pd) / max(u[a] * qd, pd, 1e-300))
        if u[a] * qd < pd:
            a += 1
        else:
            break
    qa = q[a] if a < k else np.zeros_like(p[k])
    w = np.maximum(p[a] - qa, 0.0)
    tok, s1, s2, tok2 = gumbel_draw(w, g)
    emitted = drafts[:a] + [tok] + [-1] * (k - a)
    return SampledResult(a, emitted, tok, float(margin), s1 - s2,
                         ((p[a, tok], qa[tok]), (p[a, tok2], qa[tok2])))
