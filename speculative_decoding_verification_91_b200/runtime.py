"""Device-side state for the verify step: weights, paged cache pools,
workspace and the spec_model descriptor handed to the C ABI.

PyTorch provides device memory and streams here; all arithmetic of the
verify step runs in libspecverify.so.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import binding as B

BF16_NAN = 0x7FC0


def to_device_bf16(bits: np.ndarray, device) -> torch.Tensor:
    """Upload bf16 bit patterns (numpy uint16) as a bfloat16 tensor."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device=device, non_blocking=False).view(torch.bfloat16)


@dataclass
class LayerConfig:
    window: int
    kv_equal: bool
    rope_fraction: float
    split_tokens: int = 0      # 0: the model's split


class DeviceModel:
    """Weights and cache pools of one synthetic target on one GPU.

    Pools are allocated for num_pages pages and filled with bf16 NaN when
    `poison` is set, so that any read of a slot that was never written shows
    up in the results."""

    def __init__(self, *, d_model, n_q_heads, n_kv_heads, head_dim, vocab, layers, w_lm_bits,
                 layer_weights, num_pages, split_tokens, rope_theta=10000.0, rms_eps=1e-6,
                 device="cuda", poison=True, w_emb_bits=None):
        self.device = torch.device(device)
        self.d_model, self.n_q_heads, self.n_kv_heads = d_model, n_q_heads, n_kv_heads
        self.head_dim, self.vocab, self.num_pages = head_dim, vocab, num_pages
        self.layers = list(layers)
        self.w_lm = to_device_bf16(w_lm_bits, self.device)
        self.w_emb = self.w_lm if w_emb_bits is None else to_device_bf16(w_emb_bits, self.device)
        self.w_qkv, self.w_o, self.k_pool, self.v_pool, self.ksb_pool = [], [], [], [], []
        P, H, D = num_pages, n_kv_heads, head_dim
        for (wqkv, wo), spec in zip(layer_weights, self.layers):
            self.w_qkv.append(to_device_bf16(wqkv, self.device))
            self.w_o.append(to_device_bf16(wo, self.device))
            n_rot = int(round(spec.rope_fraction * D / 2))
            self.k_pool.append(self._pool((P, H, B.SPEC_PAGE_SIZE, D), poison))
            if spec.kv_equal:
                self.v_pool.append(None)
                self.ksb_pool.append(self._pool((P, H, B.SPEC_PAGE_SIZE, 2 * n_rot), poison))
            else:
                self.v_pool.append(self._pool((P, H, B.SPEC_PAGE_SIZE, D), poison))
                self.ksb_pool.append(None)
        self._layers_c = (B.SpecLayer * len(self.layers))()
        for l, spec in enumerate(self.layers):
            self._layers_c[l] = B.SpecLayer(
                self.w_qkv[l].data_ptr(), self.w_o[l].data_ptr(), self.k_pool[l].data_ptr(),
                self.v_pool[l].data_ptr() if self.v_pool[l] is not None else None,
                self.ksb_pool[l].data_ptr() if self.ksb_pool[l] is not None else None,
                int(spec.window), int(spec.kv_equal), float(spec.rope_fraction),
                int(spec.split_tokens))
        self.desc = B.SpecModel(len(self.layers), d_model, n_q_heads, n_kv_heads, head_dim, vocab,
                                B.SPEC_PAGE_SIZE, num_pages, split_tokens, float(rope_theta),
                                float(rms_eps), self.w_lm.data_ptr(), self.w_emb.data_ptr(),
                                ctypes.cast(self._layers_c, ctypes.POINTER(B.SpecLayer)))

    def _pool(self, shape, poison):
        if poison:
            return torch.full(shape, BF16_NAN, dtype=torch.int16, device=self.device).view(torch.bfloat16)
        return torch.empty(shape, dtype=torch.bfloat16, device=self.device)

    def pool_bytes(self) -> int:
        n = 0
        for l in range(len(self.layers)):
            for which in range(3):
                n += B.spec_layer_pool_bytes(self.desc, l, which)
        return n


class Workspace:
    """Caller-owned scratch for the kernels, cleared once at creation."""

    def __init__(self, nbytes: int, device="cuda", stream=None):
        if nbytes <= 0:
            raise ValueError("workspace size must be positive (check the model / batch limits)")
        self.nbytes = int(nbytes)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        B.spec_workspace_init(self.buf, self.nbytes, stream)

    def ptr(self) -> int:
        return self.buf.data_ptr()

    def device_status(self, stream=None) -> int:
        return B.spec_read_device_status(self.buf, self.nbytes, stream)


class DeviceDrafter:
    """Weights of one synthetic MTP drafter on one GPU and its spec_drafter
    descriptor.  blocks: (w_q bits, w_o bits, target layer) per block."""

    def __init__(self, *, d_draft, n_q_heads, w_emb_bits, w_down_bits, w_up_bits, blocks,
                 device="cuda", clusters=None):
        self.device = torch.device(device)
        self.d_draft, self.n_q_heads = d_draft, n_q_heads
        self.w_emb = to_device_bf16(w_emb_bits, self.device)
        self.w_down = to_device_bf16(w_down_bits, self.device)
        self.w_up = to_device_bf16(w_up_bits, self.device)
        self.w_q = [to_device_bf16(b[0], self.device) for b in blocks]
        self.w_o = [to_device_bf16(b[1], self.device) for b in blocks]
        self.target_layers = [int(b[2]) for b in blocks]
        self._blocks_c = (B.SpecDraftBlock * len(blocks))()
        for i in range(len(blocks)):
            self._blocks_c[i] = B.SpecDraftBlock(self.w_q[i].data_ptr(), self.w_o[i].data_ptr(),
                                                 self.target_layers[i])
        self.clusters = clusters
        self.desc = B.SpecDrafter(d_draft, n_q_heads, len(blocks), self.w_emb.data_ptr(),
                                  self.w_down.data_ptr(), self.w_up.data_ptr(),
                                  ctypes.cast(self._blocks_c, ctypes.POINTER(B.SpecDraftBlock)),
                                  ctypes.pointer(clusters.desc) if clusters is not None else None)


class DeviceClusters:
    """Token-cluster tables of the cheap unembedding on one GPU and their
    spec_clusters descriptor."""

    def __init__(self, *, cluster_tokens, centroid_bits, clustered_bits, n_select, device="cuda"):
        self.device = torch.device(device)
        C, S = cluster_tokens.shape
        self.tokens = torch.from_numpy(np.ascontiguousarray(cluster_tokens, dtype=np.int32)).to(self.device)
        self.centroids = to_device_bf16(centroid_bits, self.device)
        self.w_clustered = to_device_bf16(clustered_bits, self.device)
        self.desc = B.SpecClusters(int(C), int(S), int(n_select), self.centroids.data_ptr(),
                                   self.tokens.data_ptr(), self.w_clustered.data_ptr())
