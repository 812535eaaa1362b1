"""Pins of the CPU oracle to facts other than itself (CPU only).

Each test checks an oracle function against what the pages state (golden
fixtures), a closed form, a special case that reduces to a textbook or
library routine (torch CPU), or brute force on tiny inputs.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_91_b200.inputs import gen
from speculative_decoding_verification_91_b200.inputs import workloads as W

from . import harness

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- formats

def test_bf16_rounding_matches_torch():
    x = np.concatenate([_rng().standard_normal(100_000) * 10.0 ** _rng(1).integers(-8, 8, 100_000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.001953125, 1.005859375, 3.4e38, -3.4e38,
                         1e-40, np.inf, -np.inf]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = oracle.bf16(x)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.isnan(oracle.bf16(np.float32(np.nan)))


def test_bf16_bits_roundtrip():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_from_bits(bits)
    finite = np.isfinite(vals)
    assert np.array_equal(oracle.bits_from_bf16(vals[finite]), bits[finite])
    assert np.array_equal(vals, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy(),
                          equal_nan=True)


# ---------------------------------------------------------------- rmsnorm

def test_rmsnorm_closed_forms():
    x = np.array([[3.0, 4.0]])
    np.testing.assert_allclose(oracle.rmsnorm(x, 0.0), x / math.sqrt(12.5), rtol=1e-15)
    y = oracle.rmsnorm(_rng().standard_normal((7, 300)), 1e-6)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-6)
    # eps matters exactly as sqrt(ms / (ms + eps)) on the output RMS
    z = np.full((1, 4), 1e-3)
    out = oracle.rmsnorm(z, 1e-6)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2)), math.sqrt(1e-6 / (1e-6 + 1e-6)), rtol=1e-12)


def test_rmsnorm_matches_torch_layer():
    x = _rng(3).standard_normal((5, 64))
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, 1e-6), ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- RoPE

def _rope64(x, pos, D, theta, frac):
    """Same rotation through complex multiplication (independent formulation):
    z_i = x_i + 1j*x_{i+D/2} times exp(1j * pos * theta_i) for rotated pairs."""
    n = oracle.rope_rotated_pairs(D, frac)
    h = D // 2
    z = x[..., :h] + 1j * x[..., h:]
    ang = np.asarray(pos, np.float64)[:, None] * (theta ** (-np.arange(h) * 2.0 / D))[None, :]
    rot = np.where(np.arange(h)[None, :] < n, np.exp(1j * ang), 1.0)
    z = z * rot[:, None, :]
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("D,frac", [(128, 1.0), (256, 0.25), (256, 1.0), (16, 0.5)])
def test_rope_equals_complex_rotation(D, frac):
    x = oracle.bf16(_rng(D).standard_normal((9, 3, D))).astype(np.float32)
    pos = np.array([0, 1, 2, 63, 64, 1023, 8191, 32768, 131071])
    got = oracle.rope(x, pos, D, 10000.0, frac).astype(np.float64)
    want = _rope64(x.astype(np.float64), pos, D, 10000.0, frac)
    np.testing.assert_allclose(got, want, rtol=0, atol=4e-6 * np.abs(x).max())


def test_rope_p0_identity_and_pos0_identity():
    x = _rng(1).standard_normal((4, 2, 64)).astype(np.float32)
    assert np.array_equal(oracle.rope(x, np.arange(4) + 100, 64, 1e4, 0.0), x)
    assert np.array_equal(oracle.rope(x, np.zeros(4, np.int64), 64, 1e4, 1.0), x)


def test_p_rope_rotates_only_highest_frequency_quarter():
    D = 256
    n = oracle.rope_rotated_pairs(D, 0.25)
    assert n == 32
    inv = oracle.rope_inv_freq(D)
    assert inv[0] == 1.0 and np.all(np.diff(inv) < 0)            # pair 0 turns fastest
    x = _rng(2).standard_normal((3, 1, D)).astype(np.float32)
    y = oracle.rope(x, np.array([5, 77, 1000]), D, 1e4, 0.25)
    changed = np.any(y != x, axis=(0, 1))
    assert set(np.nonzero(changed)[0]) == set(range(0, 32)) | set(range(128, 160))


def test_rope_relative_position_and_norm():
    D = 128
    q = _rng(4).standard_normal((1, 1, D))
    k = _rng(5).standard_normal((1, 1, D))
    for frac in (1.0, 0.25):
        dots = []
        for shift in (0, 17, 5000):
            qr = _rope64(q, [40 + shift], D, 1e4, frac)
            kr = _rope64(k, [3 + shift], D, 1e4, frac)
            dots.append(float(np.sum(qr * kr)))
            assert abs(np.linalg.norm(qr) - np.linalg.norm(q)) < 1e-12
        np.testing.assert_allclose(dots, dots[0], rtol=1e-9)
        # and the oracle's binary32 rotation agrees with it
        qo = oracle.rope(q.astype(np.float32), np.array([57]), D, 1e4, frac)
        np.testing.assert_allclose(qo, _rope64(q.astype(np.float32).astype(np.float64), [57], D, 1e4,
                                               frac), atol=1e-5)


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v, mask, scale):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=torch.from_numpy(mask)[None, None], scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("window", [0, 1, 5, 40])
def test_attend_matches_torch_sdpa(window):
    r = _rng(window)
    J, R, D = 70, 5, 16
    kpos = np.arange(J)
    qpos = np.arange(J - R, J)
    q, k, v = (r.standard_normal((R, D)), r.standard_normal((J, D)), r.standard_normal((J, D)))
    mask = (kpos[None] <= qpos[:, None])
    if window:
        mask &= kpos[None] > qpos[:, None] - window
    got = oracle.attend(q, k, v, qpos, kpos, window, 0.25)
    np.testing.assert_allclose(got, _sdpa(q, k, v, mask, 0.25), rtol=1e-12, atol=1e-13)


def test_attend_special_cases():
    r = _rng(9)
    D = 8
    k, v = r.standard_normal((6, D)), r.standard_normal((6, D))
    # one visible key -> its value exactly
    out = oracle.attend(r.standard_normal((1, D)), k[:1], v[:1], [0], [0], 0, 1.0)
    assert np.array_equal(out[0], v[0])
    # equal scores (q = 0) -> mean of the visible values
    out = oracle.attend(np.zeros((1, D)), k, v, [5], np.arange(6), 0, 1.0)
    np.testing.assert_allclose(out[0], v.mean(axis=0), rtol=1e-14)
    # window 1 -> own value
    out = oracle.attend(r.standard_normal((3, D)), k, v, [3, 4, 5], np.arange(6), 1, 1.0)
    np.testing.assert_allclose(out, v[3:6], rtol=1e-14)
    # window >= context -> global
    q = r.standard_normal((2, D))
    np.testing.assert_allclose(oracle.attend(q, k, v, [4, 5], np.arange(6), 6, 0.3),
                               oracle.attend(q, k, v, [4, 5], np.arange(6), 0, 0.3), rtol=1e-15)
    # two keys: logistic weights
    q = r.standard_normal((1, D))
    s = (q @ k[:2].T)[0] * 0.5
    w1 = 1.0 / (1.0 + math.exp(s[1] - s[0]))
    np.testing.assert_allclose(oracle.attend(q, k[:2], v[:2], [1], [0, 1], 0, 0.5)[0],
                               w1 * v[0] + (1 - w1) * v[1], rtol=1e-12)


def _tiny_model(kv_equal, window, frac, Hq=4, Hkv=2, D=16, d=32, V=50, seed=0):
    r = _rng(seed)
    nq = (Hq + Hkv + (0 if kv_equal else Hkv)) * D
    w = lambda *s: oracle.bf16(r.standard_normal(s) * 0.2)
    layer = oracle.LayerDef(window, kv_equal, frac, w(nq, d), w(d, Hq * D))
    wlm = oracle.bits_from_bf16(r.standard_normal((V, d)) * 0.3)
    return oracle.Model(d, Hq, Hkv, D, wlm, [layer])


@pytest.mark.parametrize("kv_equal,window,frac", [(False, 0, 1.0), (False, 7, 1.0), (True, 0, 0.25)])
def test_attention_layer_is_gqa_sdpa(kv_equal, window, frac):
    """Grouped-query attention over cache + new rows equals torch SDPA with the
    KV heads repeated per query group (repeat_interleave) and V = pre-RoPE K
    on key-equals-value layers."""
    m = _tiny_model(kv_equal, window, frac)
    r = _rng(7)
    Hq, Hkv, D, L, nq = 4, 2, 16, 20, 4
    kraw = oracle.bf16(r.standard_normal((L, Hkv, D)))
    vraw = None if kv_equal else oracle.bf16(r.standard_normal((L, Hkv, D)))
    lo = 0 if window == 0 else L - window + 1
    cache = oracle.cache_from_raw(m, 0, lo, kraw[lo:], None if vraw is None else vraw[lo:])
    qp = r.standard_normal((nq, Hq, D)).astype(np.float32)
    kp = r.standard_normal((nq, Hkv, D)).astype(np.float32)
    vp = None if kv_equal else r.standard_normal((nq, Hkv, D)).astype(np.float32)
    out, (kn, vn, kpn) = oracle.attention_layer(m, 0, cache, L, qp, kp, vp)
    pos = np.arange(L, L + nq)
    qr = oracle.bf16(_rope64(qp.astype(np.float64), pos, D, 1e4, frac))
    keys_all = oracle.bf16(_rope64(np.concatenate([kraw, kp]).astype(np.float64),
                                   np.arange(L + nq), D, 1e4, frac))
    vals_all = oracle.bf16(np.concatenate([kraw, kp]) if kv_equal else np.concatenate([vraw, vp]))
    kpos = np.arange(L + nq)
    mask = kpos[None] <= pos[:, None]
    if window:
        mask &= kpos[None] > pos[:, None] - window
    G = Hq // Hkv
    kt = torch.from_numpy(keys_all.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(vals_all.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    qt = torch.from_numpy(qr.astype(np.float64)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=1 / math.sqrt(D)).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=2e-2, atol=2e-2)       # rope factors differ in fp32 vs fp64
    assert np.mean(np.abs(out - ref)) < 2e-3


# ---------------------------------------------------------------- LM head

def test_lm_head_matches_torch_argmax():
    r = _rng(11)
    h = oracle.bf16(r.standard_normal((6, 96)))
    wb = oracle.bits_from_bf16(r.standard_normal((3000, 96)) * 0.02)
    ids, t1, t2 = oracle.lm_head_top2(h, wb, chunk=700)
    lg = torch.from_numpy(h.astype(np.float64)) @ torch.from_numpy(oracle.bf16_from_bits(wb).astype(np.float64)).T
    assert np.array_equal(ids, lg.argmax(dim=1).numpy())
    top = torch.topk(lg, 2, dim=1).values.numpy()
    np.testing.assert_allclose(t1, top[:, 0], rtol=1e-7)
    np.testing.assert_allclose(t2, top[:, 1], rtol=1e-7)


def test_lm_head_ties_go_to_lowest_id():
    r = _rng(12)
    h = oracle.bf16(r.standard_normal((2, 32)))
    w = r.standard_normal((500, 32)) * 0.02
    lg = h.astype(np.float64) @ w.T
    best = int(np.argmax(lg[0]))
    w[450] = w[best]          # duplicate row, in a later chunk
    w[best + 1 if best + 1 < 450 else best - 1] = w[best]
    wb = oracle.bits_from_bf16(w)
    ids, t1, t2 = oracle.lm_head_top2(h, wb, chunk=128)
    wv = oracle.bf16_from_bits(wb).astype(np.float64)
    dup = np.nonzero(np.all(wv == wv[450], axis=1))[0]
    assert ids[0] == dup.min() and t1[0] == t2[0]


# ---------------------------------------------------------------- acceptance

def test_accept_cases_from_pages():
    for case in _golden("accept_cases.json")["cases"]:
        a, emitted, nxt = oracle.accept_longest_prefix(case["drafts"], case["target"])
        assert a == case["a"], case["cite"]
        assert emitted == case["emitted"], case["cite"]
        assert nxt == case["target"][a]
        assert sum(t >= 0 for t in emitted) == a + 1      # the target always adds one token


@pytest.mark.parametrize("k", range(0, 9))
def test_accept_brute_force_over_match_patterns(k):
    g = list(range(100, 100 + k + 1))
    for pattern in itertools.product([0, 1], repeat=k):
        drafts = [g[i] if m else g[i] + 1000 for i, m in enumerate(pattern)]
        a, emitted, nxt = oracle.accept_longest_prefix(drafts, g)
        first_wrong = next((i for i, m in enumerate(pattern) if not m), k)
        assert a == first_wrong
        assert emitted[:a + 1] == g[:a + 1] and emitted[a + 1:] == [-1] * (k - a)


def test_tokens_per_forward_accounting():
    """E[a+1] for per-token accept probability p is sum_j p^j; check the
    draft recipe reproduces it, and that the page's 2.4 tokens/forward is
    reachable with k=4 (p ~ 0.69)."""
    fx = _golden("tokens_per_forward.json")
    wl = W.get_workload("b1_ctx8k")
    rs = [W.rejection_point(wl.with_(batch=1), 0, t) for t in range(4000)]
    mean_tokens = np.mean(np.array(rs) + 1)
    p = 0.8
    assert abs(mean_tokens - sum(p ** j for j in range(wl.k + 1))) < 0.05
    ps = np.linspace(0.3, 0.99, 2000)
    e = np.array([sum(pp ** j for j in range(5)) for pp in ps])
    p24 = ps[np.argmin(np.abs(e - fx["tokens_per_forward"]))]
    assert 0.6 < p24 < 0.75


# ---------------------------------------------------------------- K=V layout

def test_key_equals_value_cache_saving_is_37_5_percent():
    fx = _golden("kv_equal_saving.json")
    for D in fx["head_dims"]:
        sep = oracle.kv_values_per_token_head(D, 1.0, False)
        kv = oracle.kv_values_per_token_head(D, fx["rope_fraction"], True)
        assert 1.0 - kv / sep == fx["saving"], fx["cite"]


def test_key_equals_value_values_are_recoverable():
    """Post-RoPE K plus the pre-RoPE rotated dims hold V = pre-RoPE K exactly."""
    m = _tiny_model(True, 0, 0.25, D=32)
    kraw = oracle.bf16(_rng(3).standard_normal((10, 2, 32)))
    c = oracle.cache_from_raw(m, 0, 0, kraw, None)
    n = oracle.rope_rotated_pairs(32, 0.25)
    side = np.concatenate([c.kpre[..., :n], c.kpre[..., 16:16 + n]], axis=-1)
    rebuilt = c.k.copy()
    rebuilt[..., :n] = side[..., :n]
    rebuilt[..., 16:16 + n] = side[..., n:]
    assert np.array_equal(rebuilt, kraw)
    assert np.array_equal(c.values(), kraw)


# ---------------------------------------------------------------- whole step / loop

def test_forward_degenerate_zero_output_projection():
    """With W_o = 0 the residual stream stays the token embedding, so the
    argmax is that of the normalised tied embedding against the LM head."""
    m = _tiny_model(False, 0, 1.0, V=300)
    m.layers[0].w_o[:] = 0
    toks = [3, 17, 250]
    cache = oracle.cache_from_raw(m, 0, 0, oracle.bf16(_rng(5).standard_normal((4, 2, 16))),
                                  oracle.bf16(_rng(6).standard_normal((4, 2, 16))))
    fw = oracle.verify_forward(m, [cache], 4, toks)
    E = torch.from_numpy(oracle.bf16_from_bits(m.w_lm_bits).astype(np.float64))
    hn = torch.nn.functional.rms_norm(E[toks], (m.d_model,), eps=1e-6)
    hn = torch.from_numpy(oracle.bf16(hn.numpy()).astype(np.float64))
    lg = hn @ E.T
    assert np.array_equal(fw.g, lg.argmax(dim=1).numpy())
    # the logit values too (an argmax alone cannot see a missing final norm,
    # which only rescales each row); binary32 rounding of each logit
    np.testing.assert_allclose(fw.top1, lg.max(dim=1).values.numpy(), rtol=1e-6)


def _loop_model(seed):
    wl = W.get_workload("small_loop").with_(name=f"pin_loop{seed}", d_model=64, n_q_heads=4,
                                            n_kv_heads=2, head_dim=16, vocab=97, weight_std=0.3,
                                            layers=(W.LayerSpec(window=6),) * 2 + (W.GLOBAL_KV,))
    return wl, harness.oracle_model(wl)


@pytest.mark.parametrize("seed", [0, 1])
def test_speculative_loop_equals_greedy_decoding(seed):
    """The pages: every emitted token is checked by the target, so the output
    equals standard decoding ("Gemma 4 发布时未包含 MTP 数据" §MTP 能快多少;
    "Accelerating Gemma 4" §5 zero quality loss).  Drafts here are greedy
    tokens corrupted at random, so acceptance, rollback and the causal mask
    inside the draft block are all exercised."""
    wl, m = _loop_model(seed)
    prompt = gen.randint(seed, "pin/prompt", 0, 12, 0, wl.vocab)
    caches, g_last, _, _ = oracle.prefill(m, prompt, chunk=5)
    n = 30
    ref, margins, _, _ = oracle.greedy_decode(m, caches, len(prompt), int(prompt[-1]), n)
    ref = [int(t) for t in ref]
    flips = gen.uniform(seed, "pin/flips", 0, 1000)
    ids = gen.randint(seed, "pin/ids", 0, 1000, 0, wl.vocab)

    def drafter(step, emitted, k):
        base = len(emitted)
        out = []
        for i in range(k):
            j = base + i                            # row i predicts emitted token base+i
            c = step * k + i
            truth = ref[j] if j < len(ref) else 0
            out.append(truth if flips[c] < 0.7 else int(ids[c]))
        return out

    for k in (1, 3, 5):
        spec, accepts = oracle.speculative_decode(m, caches, len(prompt), int(prompt[-1]), k, n,
                                                  lambda s, e, kk: drafter(s, e, kk))
        assert spec == ref
        assert any(a > 0 for a in accepts) and any(a < k for a in accepts)
        assert np.mean(accepts) > 0.3 * k * 0.7        # drafts are mostly right


def test_verify_with_k0_is_one_greedy_step():
    wl, m = _loop_model(2)
    prompt = gen.randint(2, "pin/prompt2", 0, 9, 0, wl.vocab)
    caches, _, _, _ = oracle.prefill(m, prompt)
    res = oracle.verify_step(m, caches, len(prompt), int(prompt[-1]), [])
    toks, _, _, _ = oracle.greedy_decode(m, caches, len(prompt), int(prompt[-1]), 1)
    assert res.accept_len == 0 and res.emitted == [toks[0]] and res.new_len == len(prompt) + 1


def test_prefill_chunking_does_not_change_the_cache():
    wl, m = _loop_model(3)
    prompt = gen.randint(3, "pin/prompt3", 0, 17, 0, wl.vocab)
    a, ga, _, _ = oracle.prefill(m, prompt)
    b, gb, _, _ = oracle.prefill(m, prompt, chunk=4)
    assert ga == gb
    for ca, cb in zip(a, b):
        np.testing.assert_allclose(ca.k, cb.k, atol=1e-2)
        assert np.mean(ca.k != cb.k) < 1e-2


def test_tiny_workload_draft_and_guard():
    wl = W.get_workload("tiny")
    m = harness.oracle_model(wl)
    case = harness.guarded_sequence(wl, m, 0, 256)
    res = case.result
    assert res.accept_len == case.r
    assert res.emitted[:res.accept_len] == list(case.drafts[:res.accept_len])
    assert res.new_len == 256 + res.accept_len + 1
