"""The test harness's cache snapshot (paged pools -> oracle caches), on CPU.

Oracle caches are written into mock pools in the library's layout (pages of
64 tokens in a permuted block table; post-RoPE keys, values or the
key-equals-value side-band of pre-RoPE rotated dimensions) and read back:
keys, values and pre-RoPE keys must come back bit for bit, from the window
start on sliding-window layers.
"""
import numpy as np
import torch

import oracle

from . import harness

PAGE = 64


def _model(D=32, Hkv=2, Hq=4, d=16):
    r = np.random.default_rng(0)
    w = lambda *s: oracle.bf16(r.standard_normal(s) * 0.1)
    layers = [oracle.LayerDef(40, False, 1.0, w((Hq + 2 * Hkv) * D, d), w(d, Hq * D)),
              oracle.LayerDef(0, True, 0.25, w((Hq + Hkv) * D, d), w(d, Hq * D))]
    return oracle.Model(d, Hq, Hkv, D, oracle.bits_from_bf16(w(50, d)), layers)


def _to_pool(P, Hkv, width):
    return torch.zeros((P, Hkv, PAGE, width), dtype=torch.int16)


def test_snapshot_rebuilds_the_oracle_caches():
    m = _model()
    D, Hkv, L = m.head_dim, m.n_kv_heads, 150
    r = np.random.default_rng(1)
    n_pages = (L + PAGE - 1) // PAGE
    P = n_pages + 3
    table = r.permutation(P)[:n_pages].astype(np.int32)
    pools, want = [], []
    for l, spec in enumerate(m.layers):
        kraw = oracle.bf16(r.standard_normal((L, Hkv, D)))
        vraw = None if spec.kv_equal else oracle.bf16(r.standard_normal((L, Hkv, D)))
        c = oracle.cache_from_raw(m, l, 0, kraw, vraw)
        want.append(c)
        n = oracle.rope_rotated_pairs(D, spec.rope_fraction)
        kp = _to_pool(P, Hkv, D)
        vp = None if spec.kv_equal else _to_pool(P, Hkv, D)
        sp = _to_pool(P, Hkv, 2 * n) if spec.kv_equal else None
        for pos in range(L):
            pg, sl = table[pos // PAGE], pos % PAGE
            kp[pg, :, sl, :] = torch.from_numpy(oracle.bits_from_bf16(c.k[pos]).view(np.int16))
            if spec.kv_equal:
                side = np.concatenate([c.kpre[pos][:, :n], c.kpre[pos][:, D // 2:D // 2 + n]], axis=-1)
                sp[pg, :, sl, :] = torch.from_numpy(oracle.bits_from_bf16(side).view(np.int16))
            else:
                vp[pg, :, sl, :] = torch.from_numpy(oracle.bits_from_bf16(c.v[pos]).view(np.int16))
        pools.append(tuple(None if x is None else x.view(torch.bfloat16) for x in (kp, vp, sp)))
    got = harness.snapshot_caches(m, pools, table, L, PAGE)
    for spec, g, w in zip(m.layers, got, want):
        lo = L - (spec.window - 1) if spec.window else 0
        assert g.lo == lo and g.end == L
        assert np.array_equal(oracle.bits_from_bf16(g.k), oracle.bits_from_bf16(w.k[lo:]))
        assert np.array_equal(oracle.bits_from_bf16(g.values()), oracle.bits_from_bf16(w.values()[lo:]))
