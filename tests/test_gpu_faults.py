"""Device-detected bad inputs through the fused verify step (C ABI).

A corrupt block-table entry, a committed length past the sequence's
block-table row, and a token id outside the vocabulary are each caught by the
kernels' own bounds checks: the step launches and completes without a CUDA
error, the workspace status word carries the matching SPEC_DEV_* bit, the
affected work is skipped (no cache slot outside the other sequences' new
rows changes), and every other sequence's results and cache entries are
bit-identical to a clean run of the same inputs.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import gen
from speculative_decoding_verification_91_b200.inputs import workloads as W
from speculative_decoding_verification_91_b200.session import WorkloadSession

pytestmark = pytest.mark.gpu

PAGE = B.SPEC_PAGE_SIZE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    B.lib()
    yield
    torch.cuda.synchronize()


def _pools(s):
    return [p for l in range(len(s.wl.layers))
            for p in (s.dm.k_pool[l], s.dm.v_pool[l], s.dm.ksb_pool[l]) if p is not None]


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


def _session(wl):
    s = WorkloadSession(wl)
    last = np.array([W.last_token(wl, b, 0) for b in range(wl.batch)], dtype=np.int32)
    drafts = gen.randint(wl.seed, f"{wl.name}/fault_drafts", 0, wl.batch * wl.k, 0,
                         wl.vocab).astype(np.int32).reshape(wl.batch, wl.k)
    return s, last, drafts


def _new_slots(s, table, seqs):
    """(page, slot) of the new rows L..L+k of the given sequences, for the
    rows whose block-table entry is a valid page."""
    out = set()
    for b in seqs:
        L = int(s.lens[b])
        for pos in range(L, L + s.wl.k + 1):
            if pos // PAGE < table.shape[1] and 0 <= table[b, pos // PAGE] < s.num_pages:
                out.add((int(table[b, pos // PAGE]), pos % PAGE))
    return out


def _changed_slots(before, after):
    out = set()
    for a, c in zip(before, after):
        diff = np.any(a != c, axis=(1, 3))                  # [P][slot]
        out |= {(int(p), int(t)) for p, t in zip(*np.nonzero(diff))}
    return out


def _run(s, last, drafts):
    s.set_inputs(last, drafts)
    before = [_bits(p) for p in _pools(s)]
    s.step()
    torch.cuda.synchronize()
    return before, [_bits(p) for p in _pools(s)], s.outputs(), s.ws.device_status()


@pytest.mark.parametrize("name", ["small_ragged", "small_b16"])
@pytest.mark.parametrize("fault", ["bad_page", "bad_length", "bad_token"])
def test_bad_input_is_flagged_and_contained(name, fault):
    wl = W.get_workload(name)
    clean, last, drafts = _session(wl)
    _, _, want, st_clean = _run(clean, last, drafts)
    assert st_clean == 0

    s, _, _ = _session(wl)
    table = s.block_table.cpu().numpy()
    last_f = last.copy()
    if fault == "bad_page":
        b = 1
        s.block_table[b, int(s.lens[b]) // PAGE] = s.num_pages + 7    # the page of its first new row
        bit = B.SPEC_DEV_BAD_PAGE
    elif fault == "bad_length":
        b = int(np.argmin(s.lens))                                    # shortest row: -1 entries at the end
        s.seq_lens[b] = s.max_pages * PAGE - 2                        # L + k + 1 runs past its row
        bit = B.SPEC_DEV_BAD_LENGTH
    else:
        b = 0
        last_f[b] = wl.vocab + 3
        bit = B.SPEC_DEV_BAD_TOKEN
    before, after, got, status = _run(s, last_f, drafts)

    assert status & bit, (fault, hex(status))
    others = [x for x in range(wl.batch) if x != b]
    q = wl.k + 1
    for key in ("accept_len", "new_last"):
        assert np.array_equal(np.asarray(got[key])[others], np.asarray(want[key])[others]), key
    for key in ("emitted", "target_ids", "target_max"):
        g = np.asarray(got[key]).reshape(wl.batch, q)[others]
        w = np.asarray(want[key]).reshape(wl.batch, q)[others]
        assert np.array_equal(g.view(np.uint32) if g.dtype == np.float32 else g,
                              w.view(np.uint32) if w.dtype == np.float32 else w), key
    # only the other sequences' new rows (and, for a bad token, the faulty
    # sequence's own new rows in its valid pages) may change in the pools
    allowed = _new_slots(s, table, others)
    if fault == "bad_token":
        allowed |= _new_slots(s, table, [b])
    elif fault == "bad_page":
        corrupt = int(table[b, int(s.lens[b]) // PAGE])
        allowed |= {x for x in _new_slots(s, table, [b]) if x[0] != corrupt}
    assert _changed_slots(before, after) <= allowed
    # the other sequences' new cache entries equal the clean run's
    for l in range(len(wl.layers)):
        for x in others:
            L = int(s.lens[x])
            for a, c in zip(s.read_cache(l, x, L, L + q), clean.read_cache(l, x, L, L + q)):
                if a is not None:
                    assert np.array_equal(a, c)
