"""The seeded input generator does what its definition says (CPU only)."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_91_b200.inputs import gen, workloads

MASK = (1 << 64) - 1
G = 0x9E3779B97F4A7C15


def _mix(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def _draw(seed, stream, ctr):
    key = _mix(seed ^ _mix((stream + G) & MASK))
    return _mix((key + (ctr + 1) * G) & MASK)


def test_splitmix_first_outputs_match_published_sequence():
    # SplitMix64 seeded with state 0: the state advances by G before mixing,
    # so its first outputs are mix(G), mix(2G), ... (the widely published
    # reference values for seed 0 start with 0xe220a8397b1dcdaf).
    assert _mix(G) == 0xE220A8397B1DCDAF
    assert _mix((2 * G) & MASK) == 0x6E789E6AA1B965F4


def test_raw_draws_match_python_twin():
    for seed, name in [(0, "w"), (7, "ctx"), (123456789, "x/y/z")]:
        got = gen.raw_u64(seed, name, 1000, 50)
        sid = gen.fnv1a64(name)
        want = [_draw(seed, sid, 1000 + i) for i in range(50)]
        assert [int(v) for v in got] == want


def test_fnv1a_known_vectors():
    # FNV-1a 64 test vectors (Fowler/Noll/Vo): "" and "a".
    assert gen.fnv1a64("") == 0xCBF29CE484222325
    assert gen.fnv1a64("a") == 0xAF63DC4C8601EC8C


def test_normal_is_box_muller_of_the_draws():
    n = 2000
    raw = gen.raw_u64(3, "nrm", 0, n)
    u1 = 1.0 - (raw[0::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    u2 = (raw[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(n)
    z[0::2] = r * np.cos(2 * np.pi * u2)
    z[1::2] = r * np.sin(2 * np.pi * u2)
    got = gen.normal_f32(3, "nrm", 0, n, 1.0).astype(np.float64)
    np.testing.assert_allclose(got, z.astype(np.float32), rtol=0, atol=1e-6)


def test_bf16_output_is_rne_of_f32_output():
    f = gen.normal_f32(5, "b", 17, 100_001, 0.02)
    b = gen.normal_bf16(5, "b", 17, 100_001, 0.02)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, ref)


def test_slices_are_position_independent_and_threads_do_not_matter():
    full = gen.normal_bf16(1, "s", 0, 10_000)
    part = gen.normal_bf16(1, "s", 3333, 777)
    assert np.array_equal(full[3333:3333 + 777], part)
    rows = gen.normal_bf16_rows(1, "s", 100, 5, 40, 1000)
    for r in range(5):
        assert np.array_equal(rows[r], full[100 + r * 1000:100 + r * 1000 + 40])


def test_normal_moments():
    z = gen.normal_f32(11, "m", 0, 2_000_000).astype(np.float64)
    assert abs(z.mean()) < 3e-3
    assert abs(z.var() - 1.0) < 5e-3
    assert abs(np.mean(z ** 4) - 3.0) < 3e-2          # normal kurtosis


def test_randint_range_and_uniformity():
    v = gen.randint(2, "r", 0, 200_000, 10, 20)
    assert v.min() == 10 and v.max() == 19
    counts = np.bincount(v - 10, minlength=10)
    assert np.all(np.abs(counts - 20_000) < 1000)


def test_page_assignment_is_a_permutation():
    wl = workloads.get_workload("small_ragged")
    lens = workloads.context_lengths(wl)
    total, table = workloads.page_assignment(wl, lens)
    used = table[table >= 0]
    assert sorted(used.tolist()) == list(range(total))
    for b, L in enumerate(lens):
        n = workloads.pages_needed(int(L), wl.k)
        assert np.all(table[b, :n] >= 0) and np.all(table[b, n:] == -1)


def test_context_lengths_in_range():
    for name in ["b8_ragged", "b64_6layer", "small_b16"]:
        wl = workloads.get_workload(name)
        lens = workloads.context_lengths(wl)
        assert lens.min() >= wl.ctx_lo and lens.max() <= wl.ctx_hi


@pytest.mark.parametrize("name", ["small_b1", "small_ragged", "small_b16", "tiny"])
def test_drafts_follow_recipe(name):
    wl = workloads.get_workload(name)
    greedy = np.arange(100, 100 + wl.k + 1)
    for b in range(min(wl.batch, 4)):
        drafts, r = workloads.make_drafts(wl, b, 0, greedy)
        assert 0 <= r <= wl.k
        assert np.array_equal(drafts[:r], greedy[:r])
        if r < wl.k:
            assert drafts[r] != greedy[r]


def test_context_kv_layout():
    wl = workloads.get_workload("small_b1")
    lo, k, v = workloads.context_kv(wl, 0, 0, 0, 1500)
    assert lo == 1500 - 300 + 1 and k.shape == (299, wl.n_kv_heads, wl.head_dim)
    lo2, k2, v2 = workloads.context_kv(wl, 0, 0, 1, 1500)
    assert lo2 == 0 and v2 is None and k2.shape[0] == 1500
