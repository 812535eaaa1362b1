"""ctypes binding of libspecverify.so: argument marshalling only.

Every function here has the name and argument order of the C entry point in
include/specverify.h.  Tensor arguments may be ints (device addresses),
objects with ``data_ptr()`` (torch tensors) or None (NULL).  A non-zero
status raises SpecError.  There is no fallback: if the library is missing
the import of the first entry point raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_uint, c_void_p

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspecverify.so")

SPEC_OK = 0
SPEC_EINVAL = -1
SPEC_EUNSUPPORTED = -2
SPEC_ECUDA = -3
SPEC_EDEVICE = -4
SPEC_ETIMEOUT = -5
SPEC_DEV_BAD_PAGE = 0x1
SPEC_DEV_BAD_LENGTH = 0x2
SPEC_DEV_TIMEOUT = 0x4
SPEC_DEV_BAD_TOKEN = 0x8
SPEC_MAX_K = 16
SPEC_PAGE_SIZE = 64

EXPORTED = [
    "spec_status_string", "spec_layer_pool_bytes", "spec_workspace_bytes",
    "spec_lmhead_workspace_bytes", "spec_workspace_init", "spec_read_device_status",
    "spec_cache_write", "spec_verify_attn", "spec_lmhead_argmax", "spec_accept_commit",
    "spec_verify_step", "spec_profile_start", "spec_profile_collect",
    "spec_lmhead_argmax_noalloc", "spec_prefill_workspace_bytes", "spec_prefill",
    "spec_profile_launches", "spec_profile_launches_collect", "spec_launch_count",
    "spec_draft_workspace_bytes", "spec_draft",
    "spec_cluster_unembed_workspace_bytes", "spec_cluster_unembed",
    "spec_verify_sampled_workspace_bytes", "spec_verify_step_sampled",
    "spec_noalloc_read_status", "spec_noalloc_inject_status",
]
SPEC_MAX_PREFILL = 256
SPEC_NOALLOC_MAX_ROWS = 64


class SpecError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status} ({status_string(status)})")


class SpecLayer(ctypes.Structure):
    _fields_ = [
        ("w_qkv", c_void_p), ("w_o", c_void_p),
        ("k_pool", c_void_p), ("v_pool", c_void_p), ("ksb_pool", c_void_p),
        ("window", c_int), ("kv_equal", c_int), ("rope_fraction", c_float),
        ("split_tokens", c_int),
    ]


class SpecModel(ctypes.Structure):
    _fields_ = [
        ("n_layers", c_int), ("d_model", c_int), ("n_q_heads", c_int), ("n_kv_heads", c_int),
        ("head_dim", c_int), ("vocab", c_int), ("page_size", c_int), ("num_pages", c_int),
        ("split_tokens", c_int), ("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_double),
        ("w_lm", c_void_p), ("w_embed", c_void_p), ("layers", POINTER(SpecLayer)),
    ]


class SpecDraftBlock(ctypes.Structure):
    _fields_ = [("w_q", c_void_p), ("w_o", c_void_p), ("target_layer", c_int)]


class SpecClusters(ctypes.Structure):
    _fields_ = [
        ("n_clusters", c_int), ("cluster_size", c_int), ("n_select", c_int),
        ("centroids", c_void_p), ("cluster_tokens", c_void_p), ("w_clustered", c_void_p),
    ]


class SpecDrafter(ctypes.Structure):
    _fields_ = [
        ("d_draft", c_int), ("n_q_heads", c_int), ("n_blocks", c_int),
        ("w_embed", c_void_p), ("w_down", c_void_p), ("w_up", c_void_p),
        ("blocks", POINTER(SpecDraftBlock)), ("clusters", POINTER(SpecClusters)),
    ]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m speculative_decoding_verification_91_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        pm = POINTER(SpecModel)
        L.spec_status_string.restype = ctypes.c_char_p
        L.spec_status_string.argtypes = [c_int]
        L.spec_layer_pool_bytes.restype = c_size_t
        L.spec_layer_pool_bytes.argtypes = [pm, c_int, c_int]
        L.spec_workspace_bytes.restype = c_size_t
        L.spec_workspace_bytes.argtypes = [pm, c_int, c_int, c_int]
        L.spec_lmhead_workspace_bytes.restype = c_size_t
        L.spec_lmhead_workspace_bytes.argtypes = [c_int, c_int]
        L.spec_workspace_init.argtypes = [c_void_p, c_size_t, c_void_p]
        L.spec_read_device_status.argtypes = [c_void_p, c_size_t, c_void_p, POINTER(c_uint)]
        L.spec_cache_write.argtypes = [pm, c_int, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                                       c_void_p]
        L.spec_verify_attn.argtypes = [pm, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                       c_void_p, c_int, c_int, c_void_p, c_void_p, c_size_t,
                                       c_void_p]
        L.spec_lmhead_argmax.argtypes = [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                         c_void_p, c_void_p, c_size_t, c_void_p]
        L.spec_accept_commit.argtypes = [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p]
        L.spec_verify_step.argtypes = [pm, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_size_t, c_void_p]
        L.spec_lmhead_argmax_noalloc.argtypes = [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                                 c_void_p, c_void_p]
        L.spec_noalloc_read_status.argtypes = [c_void_p, POINTER(c_uint)]
        L.spec_noalloc_inject_status.argtypes = [c_uint, c_void_p]
        L.spec_prefill_workspace_bytes.restype = c_size_t
        L.spec_prefill_workspace_bytes.argtypes = [pm, c_int, c_int, c_int]
        L.spec_prefill.argtypes = [pm, c_void_p, c_int, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                   c_void_p, c_void_p, c_size_t, c_void_p]
        L.spec_profile_launches.argtypes = [c_int]
        L.spec_profile_launches_collect.argtypes = [POINTER(c_float), c_int, POINTER(c_int)]
        L.spec_profile_start.argtypes = [c_int]
        L.spec_profile_collect.argtypes = [POINTER(c_float), POINTER(c_float), c_int]
        pd = POINTER(SpecDrafter)
        L.spec_draft_workspace_bytes.argtypes = [pm, pd, c_int, c_int]
        L.spec_draft.argtypes = [pm, pd, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
        pc = POINTER(SpecClusters)
        L.spec_cluster_unembed_workspace_bytes.argtypes = [c_int, c_int, pc]
        L.spec_cluster_unembed.argtypes = [c_void_p, c_int, c_int, pc, c_void_p, c_void_p, c_void_p,
                                           c_size_t, c_void_p]
        L.spec_verify_sampled_workspace_bytes.argtypes = [pm, c_int, c_int, c_int]
        L.spec_verify_step_sampled.argtypes = [pm, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                               c_int, c_int, c_float, c_void_p, c_void_p, c_void_p,
                                               c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                               c_size_t, c_void_p]
        sizes = ("spec_prefill_workspace_bytes", "spec_draft_workspace_bytes",
                 "spec_cluster_unembed_workspace_bytes", "spec_verify_sampled_workspace_bytes")
        for name in EXPORTED[4:]:
            if name not in sizes:
                getattr(L, name).restype = c_int
        for name in sizes:
            getattr(L, name).restype = c_size_t
        L.spec_launch_count.argtypes = []
        L.spec_launch_count.restype = ctypes.c_ulonglong
        _lib = L
    return _lib


def _p(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _s(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> int:
    if rc != SPEC_OK:
        raise SpecError(rc, where)
    return rc


def status_string(status: int) -> str:
    return lib().spec_status_string(status).decode()


def spec_layer_pool_bytes(model: SpecModel, layer: int, which: int) -> int:
    return int(lib().spec_layer_pool_bytes(ctypes.byref(model), layer, which))


def spec_workspace_bytes(model: SpecModel, max_batch: int, max_k: int, max_pages: int) -> int:
    return int(lib().spec_workspace_bytes(ctypes.byref(model), max_batch, max_k, max_pages))


def spec_lmhead_workspace_bytes(M: int, V: int) -> int:
    return int(lib().spec_lmhead_workspace_bytes(M, V))


def spec_workspace_init(ws, ws_bytes: int, stream=None) -> int:
    return _check(lib().spec_workspace_init(_p(ws), ws_bytes, _s(stream)), "spec_workspace_init")


def spec_read_device_status(ws, ws_bytes: int, stream=None) -> int:
    """Returns the SPEC_DEV_* bits (and clears them); never raises on bits."""
    v = c_uint(0)
    rc = lib().spec_read_device_status(_p(ws), ws_bytes, _s(stream), ctypes.byref(v))
    if rc not in (SPEC_OK, SPEC_EDEVICE, SPEC_ETIMEOUT):
        raise SpecError(rc, "spec_read_device_status")
    return int(v.value)


def spec_cache_write(model, layer, block_table_row, max_pages, pos0, n_tok, k_raw, v_raw,
                     stream=None) -> int:
    return _check(lib().spec_cache_write(ctypes.byref(model), layer, _p(block_table_row), max_pages,
                                         pos0, n_tok, _p(k_raw), _p(v_raw), _s(stream)),
                  "spec_cache_write")


def spec_verify_attn(model, layer, q, k_new, v_new, block_table, max_pages, seq_lens, B, k, out,
                     ws, ws_bytes, stream=None) -> int:
    return _check(lib().spec_verify_attn(ctypes.byref(model), layer, _p(q), _p(k_new), _p(v_new),
                                         _p(block_table), max_pages, _p(seq_lens), B, k, _p(out),
                                         _p(ws), ws_bytes, _s(stream)), "spec_verify_attn")


def spec_lmhead_argmax(h, w, M, d, V, ids, maxlogit, ws, ws_bytes, stream=None) -> int:
    return _check(lib().spec_lmhead_argmax(_p(h), _p(w), M, d, V, _p(ids), _p(maxlogit), _p(ws),
                                           ws_bytes, _s(stream)), "spec_lmhead_argmax")


def spec_accept_commit(drafts, target, B, k, seq_lens, accept_len, emitted, last_token,
                       stream=None) -> int:
    return _check(lib().spec_accept_commit(_p(drafts), _p(target), B, k, _p(seq_lens),
                                           _p(accept_len), _p(emitted), _p(last_token), _s(stream)),
                  "spec_accept_commit")


def spec_verify_step(model, block_table, max_pages, last_token, drafts, B, k, seq_lens, accept_len,
                     emitted, new_last_token, target_ids, target_maxlogit, ws, ws_bytes,
                     stream=None) -> int:
    return _check(lib().spec_verify_step(ctypes.byref(model), _p(block_table), max_pages,
                                         _p(last_token), _p(drafts), B, k, _p(seq_lens),
                                         _p(accept_len), _p(emitted), _p(new_last_token),
                                         _p(target_ids), _p(target_maxlogit), _p(ws), ws_bytes,
                                         _s(stream)), "spec_verify_step")



def spec_profile_start(n_steps: int) -> int:
    return _check(lib().spec_profile_start(n_steps), "spec_profile_start")


def spec_profile_collect(n_steps: int):
    """(step_ms list, lmhead_ms list) of the last n profiled steps."""
    a = (c_float * n_steps)()
    b = (c_float * n_steps)()
    _check(lib().spec_profile_collect(a, b, n_steps), "spec_profile_collect")
    return list(a), list(b)


def spec_lmhead_argmax_noalloc(h, w, M, d, V, ids, maxlogit, stream=None) -> int:
    """spec_lmhead_argmax without a workspace: the scratch is a fixed device
    array inside the library, for callers that cannot allocate device memory.
    Raises SpecError(SPEC_EUNSUPPORTED) when M > SPEC_NOALLOC_MAX_ROWS."""
    rc = lib().spec_lmhead_argmax_noalloc(_p(h), _p(w), M, d, V, _p(ids), _p(maxlogit), _s(stream))
    if rc == SPEC_EUNSUPPORTED:
        raise SpecError(rc, f"spec_lmhead_argmax_noalloc: M={M} exceeds the fixed scratch "
                            f"(M <= {SPEC_NOALLOC_MAX_ROWS})")
    return _check(rc, "spec_lmhead_argmax_noalloc")


def spec_noalloc_read_status(stream=None) -> int:
    """SPEC_DEV_* bits of spec_lmhead_argmax_noalloc's scratch (read and
    cleared; synchronises the stream); never raises on bits."""
    v = c_uint(0)
    rc = lib().spec_noalloc_read_status(_s(stream), ctypes.byref(v))
    if rc not in (SPEC_OK, SPEC_EDEVICE, SPEC_ETIMEOUT):
        raise SpecError(rc, "spec_noalloc_read_status")
    return int(v.value)


def spec_noalloc_inject_status(bits: int, stream=None) -> int:
    return _check(lib().spec_noalloc_inject_status(bits, _s(stream)), "spec_noalloc_inject_status")


def spec_prefill_workspace_bytes(model: SpecModel, max_batch: int, max_n: int, max_pages: int) -> int:
    return int(lib().spec_prefill_workspace_bytes(ctypes.byref(model), max_batch, max_n, max_pages))


def spec_prefill(model, block_table, max_pages, tokens, B, n, seq_lens, next_token, next_maxlogit,
                 ws, ws_bytes, stream=None) -> int:
    return _check(lib().spec_prefill(ctypes.byref(model), _p(block_table), max_pages, _p(tokens), B, n,
                                     _p(seq_lens), _p(next_token), _p(next_maxlogit), _p(ws),
                                     ws_bytes, _s(stream)), "spec_prefill")


def spec_profile_launches(max_marks: int = 256) -> int:
    return _check(lib().spec_profile_launches(max_marks), "spec_profile_launches")


def spec_launch_count() -> int:
    """Kernels the library has launched since it was loaded."""
    return int(lib().spec_launch_count())


def spec_profile_launches_collect(max_marks: int = 256):
    """Per-launch intervals (ms, launch order) of the profiled call."""
    buf = (c_float * max_marks)()
    n = c_int(0)
    _check(lib().spec_profile_launches_collect(buf, max_marks, ctypes.byref(n)),
           "spec_profile_launches_collect")
    return list(buf[:n.value])


def spec_draft_workspace_bytes(model, drafter, B: int, max_pages: int) -> int:
    return int(lib().spec_draft_workspace_bytes(ctypes.byref(model), ctypes.byref(drafter), B, max_pages))


def spec_draft(model, drafter, block_table, max_pages, seq_lens, prev_hidden, prev_token, B, k,
               drafts, draft_maxlogit, ws, ws_bytes, stream=None) -> int:
    return _check(lib().spec_draft(ctypes.byref(model), ctypes.byref(drafter), _p(block_table),
                                   max_pages, _p(seq_lens), _p(prev_hidden), _p(prev_token), B, k,
                                   _p(drafts), _p(draft_maxlogit), _p(ws), ws_bytes, _s(stream)),
                  "spec_draft")


def spec_cluster_unembed_workspace_bytes(M: int, d: int, clusters) -> int:
    return int(lib().spec_cluster_unembed_workspace_bytes(M, d, ctypes.byref(clusters)))


def spec_cluster_unembed(h, M, d, clusters, ids, maxlogit, ws, ws_bytes, stream=None) -> int:
    return _check(lib().spec_cluster_unembed(_p(h), M, d, ctypes.byref(clusters), _p(ids),
                                             _p(maxlogit), _p(ws), ws_bytes, _s(stream)),
                  "spec_cluster_unembed")


def spec_verify_sampled_workspace_bytes(model, B: int, k: int, max_pages: int) -> int:
    return int(lib().spec_verify_sampled_workspace_bytes(ctypes.byref(model), B, k, max_pages))


def spec_verify_step_sampled(model, block_table, max_pages, last_token, drafts, draft_logits, B, k,
                             temperature, u_accept, u_draw, seq_lens, accept_len, emitted,
                             new_last_token, target_logits, ws, ws_bytes, stream=None) -> int:
    return _check(lib().spec_verify_step_sampled(
        ctypes.byref(model), _p(block_table), max_pages, _p(last_token), _p(drafts), _p(draft_logits),
        B, k, float(temperature), _p(u_accept), _p(u_draw), _p(seq_lens), _p(accept_len),
        _p(emitted), _p(new_last_token), _p(target_logits), _p(ws), ws_bytes, _s(stream)),
        "spec_verify_step_sampled")
