"""Pins of the sampled-verification oracle (CPU only).

The pages state the property this must keep: the emitted tokens are
distributed as if the target alone had sampled them.  It is checked by
Monte Carlo on a tiny vocabulary (drafts drawn from the draft distribution,
fresh uniforms per trial), together with the Gumbel-max draw's frequencies
and the special cases p = q (every draft accepted) and p(d) = 0 (rejected).
"""
import math

import numpy as np
import pytest

from oracle import sampled as OS


def _rng(seed):
    return np.random.default_rng(seed)


def test_softmax_temperature_closed_forms():
    # logits (0, ln 2): weights 1 : 2 at T = 1, 1 : 4 at T = 1/2, 1 : sqrt 2 at T = 2
    lg = np.array([[0.0, math.log(2.0)]])
    np.testing.assert_allclose(OS.softmax(lg, 1.0), [[1 / 3, 2 / 3]], rtol=1e-15)
    np.testing.assert_allclose(OS.softmax(lg, 0.5), [[1 / 5, 4 / 5]], rtol=1e-15)
    r2 = math.sqrt(2.0)
    np.testing.assert_allclose(OS.softmax(lg, 2.0), [[1 / (1 + r2), r2 / (1 + r2)]], rtol=1e-15)
    # a common shift leaves it unchanged (up to the rounding of 1000 + ln 2);
    # large logits do not overflow
    np.testing.assert_allclose(OS.softmax(lg + 1000.0, 0.5), [[1 / 5, 4 / 5]], rtol=1e-12)


def test_full_logits_match_torch_and_the_argmax_head():
    from oracle import verify as OV
    import torch
    r = _rng(5)
    h = OV.bf16(r.standard_normal((3, 40)))
    wb = OV.bits_from_bf16(r.standard_normal((2100, 40)) * 0.05)
    lg = OS.full_logits(h, wb, chunk=512)
    ref = (torch.from_numpy(h.astype(np.float64)) @
           torch.from_numpy(OV.bf16_from_bits(wb).astype(np.float64)).T).float().numpy()
    assert lg.dtype == np.float32 and np.array_equal(lg, ref)       # each logit rounded once
    ids, top1, _ = OV.lm_head_top2(h, wb, chunk=700)
    assert np.array_equal(np.argmax(lg, axis=1), ids) and np.array_equal(lg.max(axis=1), top1)


def test_gumbel_draw_frequencies_follow_the_weights():
    r = _rng(0)
    w = np.array([0.5, 0.0, 0.2, 0.3])
    n = 40000
    counts = np.zeros(4)
    for _ in range(n):
        t, _, _, _ = OS.gumbel_draw(w, r.random(4))
        counts[t] += 1
    assert counts[1] == 0
    np.testing.assert_allclose(counts / n, w, atol=0.012)


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_emitted_tokens_follow_the_target_distribution(T):
    r = _rng(1)
    V, k, n = 5, 2, 30000
    p_logits = r.standard_normal((k + 1, V)).astype(np.float32) * 1.5
    q_logits = r.standard_normal((k, V)).astype(np.float32) * 1.5
    p = OS.softmax(p_logits, T)
    q = OS.softmax(q_logits, T)
    first = np.zeros(V)
    second = np.zeros(V)
    n_second = 0
    accepted = 0
    for _ in range(n):
        drafts = [r.choice(V, p=q[0]), r.choice(V, p=q[1])]
        res = OS.speculative_sample(p_logits, q_logits, drafts, r.random(k), r.random(V), T)
        first[res.emitted[0]] += 1
        accepted += res.accept_len
        if res.accept_len >= 1:          # token 1 followed the accepted draft 0
            second[res.emitted[1]] += 1
            n_second += 1
    np.testing.assert_allclose(first / n, p[0], atol=0.012)
    np.testing.assert_allclose(second / n_second, p[1], atol=0.02)
    assert 0 < accepted < n * k


def test_equal_distributions_accept_everything():
    r = _rng(2)
    V, k = 7, 3
    logits = r.standard_normal((k + 1, V)).astype(np.float32)
    drafts = [1, 4, 2]
    res = OS.speculative_sample(logits, logits[:k], drafts, r.random(k) * 0.999, r.random(V))
    assert res.accept_len == k and res.emitted[:k] == drafts


def test_impossible_draft_is_rejected_and_redrawn_elsewhere():
    V = 6
    p_logits = np.zeros((2, V), np.float32)
    p_logits[0, 3] = -1e4                 # the target never emits token 3 first
    q_logits = np.zeros((1, V), np.float32)
    res = OS.speculative_sample(p_logits, q_logits, [3], np.array([0.0]), _rng(3).random(V))
    assert res.accept_len == 0 and res.emitted[0] != 3 and res.emitted[1] == -1
