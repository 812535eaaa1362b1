"""A synthetic verify-step workload resident on one GPU.

Builds the device model from the seeded weights, assigns pages, writes every
sequence's context into the cache through spec_cache_write (RoPE and the
key-equals-value side-band are applied by the library), and holds the
step's input/output buffers.  Used by the benchmark and the GPU tests.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B
from .inputs import workloads as W
from .runtime import DeviceModel, LayerConfig, Workspace, to_device_bf16


class WorkloadSession:
    def __init__(self, wl: W.Workload, attempts=None, device="cuda", poison=True,
                 extra_tokens: int = 0, fill_context: bool = True, lens=None):
        self.wl = wl
        self.device = torch.device(device)
        self.lens = np.asarray(W.context_lengths(wl) if lens is None else lens, dtype=np.int64)
        self.attempts = list(attempts) if attempts is not None else [0] * wl.batch
        self.num_pages, table = W.page_assignment(wl, self.lens, extra_tokens)
        self.max_pages = table.shape[1]
        layer_w = [W.layer_weights(wl, l) for l in range(len(wl.layers))]
        self.dm = DeviceModel(
            d_model=wl.d_model, n_q_heads=wl.n_q_heads, n_kv_heads=wl.n_kv_heads,
            head_dim=wl.head_dim, vocab=wl.vocab,
            layers=[LayerConfig(s.window, s.kv_equal, s.rope_fraction, s.split_tokens)
                    for s in wl.layers],
            w_lm_bits=W.lm_head_weight(wl), w_emb_bits=W.embedding_weight(wl),
            layer_weights=layer_w, num_pages=self.num_pages,
            split_tokens=wl.split_tokens, rope_theta=wl.rope_theta, rms_eps=wl.rms_eps,
            device=self.device, poison=poison)
        del layer_w
        self.block_table = torch.from_numpy(table).to(self.device)
        if fill_context:
            for b in range(wl.batch):
                self.write_context(b, self.attempts[b])
        self.ws = Workspace(B.spec_workspace_bytes(self.dm.desc, wl.batch, wl.k, self.max_pages),
                            self.device)
        Bn, q = wl.batch, wl.q_rows
        i32 = dict(dtype=torch.int32, device=self.device)
        self.seq_lens0 = torch.tensor(self.lens, **i32)
        self.seq_lens = self.seq_lens0.clone()
        self.last_token = torch.zeros(Bn, **i32)
        self.drafts = torch.zeros(max(1, Bn * wl.k), **i32)
        self.accept_len = torch.zeros(Bn, **i32)
        self.emitted = torch.zeros(Bn * q, **i32)
        self.new_last = torch.zeros(Bn, **i32)
        self.target_ids = torch.zeros(Bn * q, **i32)
        self.target_max = torch.zeros(Bn * q, dtype=torch.float32, device=self.device)

    def write_context(self, b: int, attempt: int):
        wl = self.wl
        L = int(self.lens[b])
        for l in range(len(wl.layers)):
            lo, k, v = W.context_kv(wl, b, attempt, l, L)
            if L - lo == 0:
                continue
            kd = to_device_bf16(k, self.device)
            vd = None if v is None else to_device_bf16(v, self.device)
            B.spec_cache_write(self.dm.desc, l, self.block_table[b], self.max_pages, lo, L - lo, kd, vd)
        torch.cuda.synchronize(self.device)

    def set_inputs(self, last_tokens, drafts):
        self.last_token.copy_(torch.as_tensor(np.asarray(last_tokens, dtype=np.int32)))
        if self.wl.k > 0:
            self.drafts.copy_(torch.as_tensor(np.asarray(drafts, dtype=np.int32).reshape(-1)))

    def reset_lengths(self):
        self.seq_lens.copy_(self.seq_lens0)

    def step(self, stream=None, with_targets=True, k=None):
        """One spec_verify_step with this session's inputs (k defaults to the
        workload's; any k up to it fits the workspace)."""
        wl = self.wl
        k = wl.k if k is None else k
        B.spec_verify_step(self.dm.desc, self.block_table, self.max_pages, self.last_token,
                           self.drafts if k > 0 else None, wl.batch, k, self.seq_lens,
                           self.accept_len, self.emitted, self.new_last,
                           self.target_ids if with_targets else None,
                           self.target_max if with_targets else None,
                           self.ws.buf, self.ws.nbytes, stream)

    def step_one(self, b: int, stream=None, with_targets=True):
        """One batch-1 spec_verify_step on sequence slot b alone (its block-table
        row, length, inputs and outputs; the workspace is shared)."""
        wl = self.wl
        k, q = wl.k, wl.q_rows
        B.spec_verify_step(self.dm.desc, self.block_table[b], self.max_pages, self.last_token[b:b + 1],
                           self.drafts[b * k:(b + 1) * k] if k > 0 else None, 1, k,
                           self.seq_lens[b:b + 1], self.accept_len[b:b + 1],
                           self.emitted[b * q:(b + 1) * q], self.new_last[b:b + 1],
                           self.target_ids[b * q:(b + 1) * q] if with_targets else None,
                           self.target_max[b * q:(b + 1) * q] if with_targets else None,
                           self.ws.buf, self.ws.nbytes, stream)

    # ---------------------------------------------------------------- prefill

    def prefill(self, tokens: np.ndarray, chunk: int = 256):
        """Prefill tokens [B][n] from the current lengths through spec_prefill
        in chunks; returns (next_token [B], its logit [B]) after the last chunk."""
        tokens = np.asarray(tokens, dtype=np.int32)
        Bn, n = tokens.shape
        chunk = min(chunk, B.SPEC_MAX_PREFILL)
        if not hasattr(self, "pws"):
            nb = B.spec_prefill_workspace_bytes(self.dm.desc, self.wl.batch, chunk, self.max_pages)
            from .runtime import Workspace
            self.pws = Workspace(nb, self.device)
        nxt = torch.zeros(Bn, dtype=torch.int32, device=self.device)
        nmax = torch.zeros(Bn, dtype=torch.float32, device=self.device)
        dev_tok = torch.from_numpy(tokens).to(self.device)
        for c0 in range(0, n, chunk):
            c = min(chunk, n - c0)
            part = dev_tok[:, c0:c0 + c].contiguous()
            B.spec_prefill(self.dm.desc, self.block_table, self.max_pages, part, Bn, c, self.seq_lens,
                           nxt, nmax, self.pws.buf, self.pws.nbytes)
        torch.cuda.synchronize(self.device)
        return nxt.cpu().numpy(), nmax.cpu().numpy()

    # ---------------------------------------------------------------- loops

    def greedy(self, last: np.ndarray, n_tokens: int):
        """k = 0 verify steps: one token per step.  Returns tokens [B][n] and
        the max logit of every step."""
        toks = np.zeros((self.wl.batch, n_tokens), dtype=np.int64)
        maxes = np.zeros((self.wl.batch, n_tokens), dtype=np.float32)
        cur = np.asarray(last, dtype=np.int32)
        for t in range(n_tokens):
            self.last_token.copy_(torch.from_numpy(cur))
            self.step(k=0)
            o = self.outputs()
            toks[:, t] = o["target_ids"][:, 0]
            maxes[:, t] = o["target_max"][:, 0]
            cur = o["new_last"].astype(np.int32)
        return toks, maxes

    def speculative(self, last: np.ndarray, n_steps: int, drafter):
        """n_steps verify steps of k drafts each; drafter(step, emitted_b,
        b) -> k drafts for sequence b given its emitted tokens so far.
        Returns (emitted streams per sequence, accept lengths [steps][B])."""
        wl = self.wl
        streams = [[] for _ in range(wl.batch)]
        accepts = []
        cur = np.asarray(last, dtype=np.int32)
        for st in range(n_steps):
            d = np.stack([np.asarray(drafter(st, streams[b], b), dtype=np.int32)
                          for b in range(wl.batch)])
            self.set_inputs(cur, d)
            self.step()
            o = self.outputs()
            for b in range(wl.batch):
                a = int(o["accept_len"][b])
                streams[b].extend(int(t) for t in o["emitted"][b][:a + 1])
            accepts.append(o["accept_len"].copy())
            cur = o["new_last"].astype(np.int32)
        return streams, np.array(accepts)

    def outputs(self):
        torch.cuda.synchronize(self.device)
        q = self.wl.q_rows
        return dict(
            accept_len=self.accept_len.cpu().numpy(),
            emitted=self.emitted.cpu().numpy().reshape(-1, q),
            new_last=self.new_last.cpu().numpy(),
            seq_lens=self.seq_lens.cpu().numpy(),
            target_ids=self.target_ids.cpu().numpy().reshape(-1, q),
            target_max=self.target_max.cpu().numpy().reshape(-1, q),
        )

    def read_cache(self, l: int, b: int, lo: int, hi: int):
        """(k, v, ksb) bf16 bit patterns of positions [lo, hi) of sequence b."""
        table = self.block_table[b].cpu().numpy()
        out = []
        for pool in (self.dm.k_pool[l], self.dm.v_pool[l], self.dm.ksb_pool[l]):
            if pool is None:
                out.append(None)
                continue
            rows = []
            for pos in range(lo, hi):
                pg = int(table[pos // B.SPEC_PAGE_SIZE])
                rows.append(pool[pg, :, pos % B.SPEC_PAGE_SIZE, :])
            t = torch.stack(rows) if rows else pool[:0, :, 0, :]
            out.append(t.view(torch.int16).cpu().numpy().view(np.uint16))
        return tuple(out)
