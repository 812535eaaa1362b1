"""The C-ABI library builds, loads and exports what include/specverify.h
declares; host-side validation and layout queries work without a GPU."""
import ctypes
import os
import re

import pytest

from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "specverify.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return B.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ \*]*?\b(spec_[a-z_]+)\s*\(",
                                 text, flags=re.M)))


def test_every_declared_function_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(B.EXPORTED)


def test_status_strings(lib):
    assert B.status_string(0) == "ok"
    assert "invalid" in B.status_string(-1)
    assert B.status_string(12345) == "unknown status"


FAKE = 0x10000  # 16-byte aligned dummy address; never dereferenced on the host paths tested


def _model(kv_equal=True, D=256, frac=0.25, num_pages=100, n_layers=1):
    layers = (B.SpecLayer * n_layers)()
    for l in range(n_layers):
        layers[l] = B.SpecLayer(FAKE, FAKE, FAKE, None if kv_equal else FAKE, FAKE if kv_equal else None,
                                0, int(kv_equal), frac, 0)
    m = B.SpecModel(n_layers, 2560, 16, 8, D, 262144, 64, num_pages, 256, 10000.0, 1e-6, FAKE, FAKE,
                    ctypes.cast(layers, ctypes.POINTER(B.SpecLayer)))
    m._keep = layers
    return m


def test_key_equals_value_pool_is_37_5_percent_smaller(lib):
    kv = _model(True)
    sep = _model(False, frac=1.0)
    kv_bytes = sum(B.spec_layer_pool_bytes(kv, 0, w) for w in range(3))
    sep_bytes = sum(B.spec_layer_pool_bytes(sep, 0, w) for w in range(3))
    assert kv_bytes == 100 * 8 * 64 * (256 + 64) * 2
    assert 1 - kv_bytes / sep_bytes == 0.375
    assert B.spec_layer_pool_bytes(kv, 0, 1) == 0 and B.spec_layer_pool_bytes(sep, 0, 2) == 0


def test_workspace_sizes(lib):
    m = _model()
    ws = B.spec_workspace_bytes(m, 8, 4, 520)
    assert ws > 4096
    assert B.spec_workspace_bytes(m, 8, 17, 520) == 0      # k above the limit
    assert B.spec_workspace_bytes(m, 0, 4, 520) == 0
    assert B.spec_workspace_bytes(m, 16, 4, 520) > ws
    assert B.spec_lmhead_workspace_bytes(5, 262144) > 4096


def test_invalid_arguments_are_rejected_before_any_launch(lib):
    m = _model()
    L = lib
    pm = ctypes.byref(m)
    # null workspace / pointers
    assert L.spec_verify_step(pm, FAKE, 10, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, FAKE, None, None,
                              None, 0, None) == B.SPEC_EINVAL
    # k out of range
    assert L.spec_verify_step(pm, FAKE, 10, FAKE, FAKE, 1, 17, FAKE, FAKE, FAKE, FAKE, None, None,
                              FAKE, 1 << 30, None) == B.SPEC_EINVAL
    # drafts missing with k > 0
    assert L.spec_verify_step(pm, FAKE, 10, FAKE, None, 1, 2, FAKE, FAKE, FAKE, FAKE, None, None,
                              FAKE, 1 << 30, None) == B.SPEC_EINVAL
    # workspace too small
    assert L.spec_verify_step(pm, FAKE, 10, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, FAKE, None, None,
                              FAKE, 100, None) == B.SPEC_EINVAL
    # misaligned LM head weights
    assert L.spec_lmhead_argmax(FAKE, FAKE + 2, 4, 512, 1000, FAKE, None, FAKE, 1 << 20,
                                None) == B.SPEC_EINVAL
    assert L.spec_lmhead_argmax(FAKE, FAKE, 4, 511, 1000, FAKE, None, FAKE, 1 << 20,
                                None) == B.SPEC_EINVAL
    assert L.spec_accept_commit(None, FAKE, 1, 4, FAKE, FAKE, FAKE, FAKE, None) == B.SPEC_EINVAL
    assert L.spec_cache_write(pm, 0, FAKE, 2, 100, 60, FAKE, None, None) == B.SPEC_EINVAL


def test_empty_batches_are_invalid_arguments(lib):
    m = _model()
    pm = ctypes.byref(m)
    assert lib.spec_verify_step(pm, FAKE, 10, FAKE, FAKE, 0, 4, FAKE, FAKE, FAKE, FAKE, None, None,
                                FAKE, 1 << 30, None) == B.SPEC_EINVAL
    assert lib.spec_lmhead_argmax(FAKE, FAKE, 0, 512, 1000, FAKE, None, FAKE, 1 << 20,
                                  None) == B.SPEC_EINVAL
    assert lib.spec_lmhead_argmax(FAKE, FAKE, 4, 512, 0, FAKE, None, FAKE, 1 << 20,
                                  None) == B.SPEC_EINVAL
    assert lib.spec_accept_commit(FAKE, FAKE, 0, 4, FAKE, FAKE, FAKE, FAKE, None) == B.SPEC_EINVAL
    assert lib.spec_verify_attn(pm, 0, FAKE, FAKE, FAKE, FAKE, 10, FAKE, 0, 4, FAKE, FAKE, 1 << 30,
                                None) == B.SPEC_EINVAL
    assert lib.spec_workspace_bytes(pm, 0, 4, 10) == 0
    assert lib.spec_lmhead_workspace_bytes(0, 1000) == 0


def test_unsupported_shapes_are_reported(lib):
    m = _model(D=192)
    assert lib.spec_verify_step(ctypes.byref(m), FAKE, 10, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, FAKE,
                                None, None, FAKE, 1 << 30, None) == B.SPEC_EUNSUPPORTED
    m2 = _model(kv_equal=True, frac=0.5)          # side-band wider than the 64-wide tile
    assert lib.spec_verify_step(ctypes.byref(m2), FAKE, 10, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, FAKE,
                                None, None, FAKE, 1 << 30, None) == B.SPEC_EUNSUPPORTED
    m3 = _model()
    m3.page_size = 32
    assert lib.spec_verify_step(ctypes.byref(m3), FAKE, 10, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, FAKE,
                                None, None, FAKE, 1 << 30, None) == B.SPEC_EUNSUPPORTED


def _drafter(n_q_heads=16, target=0, d_draft=256):
    blocks = (B.SpecDraftBlock * 4)(*[B.SpecDraftBlock(FAKE, FAKE, target) for _ in range(4)])
    d = B.SpecDrafter(d_draft, n_q_heads, 4, FAKE, FAKE, FAKE,
                      ctypes.cast(blocks, ctypes.POINTER(B.SpecDraftBlock)))
    d._keep = blocks
    return d


def test_drafter_workspace_and_validation(lib):
    m = _model()
    d = _drafter()
    ws = B.spec_draft_workspace_bytes(m, d, 4, 520)
    assert ws > 4096
    assert B.spec_draft_workspace_bytes(m, d, 8, 520) > ws
    assert B.spec_draft_workspace_bytes(m, _drafter(n_q_heads=12), 4, 520) == 0   # not a multiple of Hkv
    assert B.spec_draft_workspace_bytes(m, _drafter(target=5), 4, 520) == 0       # no such target layer
    assert B.spec_draft_workspace_bytes(m, _drafter(d_draft=250), 4, 520) == 0
    pm, pd = ctypes.byref(m), ctypes.byref(d)
    # missing pointers, negative k, workspace too small: rejected before any launch
    assert lib.spec_draft(pm, pd, None, 10, FAKE, FAKE, FAKE, 1, 4, FAKE, None, FAKE, 1 << 30,
                          None) == B.SPEC_EINVAL
    assert lib.spec_draft(pm, pd, FAKE, 10, FAKE, FAKE, FAKE, 1, -1, FAKE, None, FAKE, 1 << 30,
                          None) == B.SPEC_EINVAL
    assert lib.spec_draft(pm, pd, FAKE, 10, FAKE, FAKE, FAKE, 1, 4, FAKE, None, FAKE, 100,
                          None) == B.SPEC_EINVAL
    assert lib.spec_draft(pm, ctypes.byref(_drafter(n_q_heads=12)), FAKE, 10, FAKE, FAKE, FAKE, 1, 4,
                          FAKE, None, FAKE, 1 << 30, None) == B.SPEC_EINVAL


def test_cluster_unembed_validation(lib):
    t = B.SpecClusters(2048, 128, 32, FAKE, FAKE, FAKE)
    assert B.spec_cluster_unembed_workspace_bytes(4, 2560, t) > 4096
    assert B.spec_cluster_unembed_workspace_bytes(4, 2561, t) == 0          # d not a multiple of 8
    assert B.spec_cluster_unembed_workspace_bytes(4, 2560, B.SpecClusters(16, 8, 17, FAKE, FAKE, FAKE)) == 0
    assert B.spec_cluster_unembed_workspace_bytes(4, 2560, B.SpecClusters(9000, 8, 4, FAKE, FAKE, FAKE)) == 0
    assert lib.spec_cluster_unembed(FAKE, 4, 2560, ctypes.byref(t), FAKE, None, FAKE, 100,
                                    None) == B.SPEC_EINVAL                   # workspace too small
    assert lib.spec_cluster_unembed(FAKE + 2, 4, 2560, ctypes.byref(t), FAKE, None, FAKE, 1 << 30,
                                    None) == B.SPEC_EINVAL                   # misaligned h
    big = B.SpecClusters(9000, 8, 4, FAKE, FAKE, FAKE)
    assert lib.spec_cluster_unembed(FAKE, 4, 2560, ctypes.byref(big), FAKE, None, FAKE, 1 << 30,
                                    None) == B.SPEC_EUNSUPPORTED


def test_sampled_verify_validation(lib):
    m = _model()
    pm = ctypes.byref(m)
    assert B.spec_verify_sampled_workspace_bytes(m, 8, 4, 520) > B.spec_workspace_bytes(m, 8, 4, 520)
    assert B.spec_verify_sampled_workspace_bytes(m, 8, 17, 520) == 0
    args = lambda T, ws_bytes, dl=FAKE: (pm, FAKE, 10, FAKE, FAKE, dl, 1, 4, ctypes.c_float(T), FAKE,
                                         FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, ws_bytes, None)
    assert lib.spec_verify_step_sampled(*args(0.0, 1 << 40)) == B.SPEC_EINVAL       # temperature
    assert lib.spec_verify_step_sampled(*args(float("nan"), 1 << 40)) == B.SPEC_EINVAL
    assert lib.spec_verify_step_sampled(*args(1.0, 1 << 40, dl=None)) == B.SPEC_EINVAL   # draft logits
    assert lib.spec_verify_step_sampled(*args(1.0, 100)) == B.SPEC_EINVAL            # workspace
