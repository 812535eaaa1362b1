"""Benchmark of the fused verify step (spec_verify_step) on synthetic inputs.

Default workload: batch 1, 8192-token context, k = 4 drafts, two layers (a
1024-token sliding-window layer with separate K/V and a key-equals-value
global layer with p-RoPE p = 0.25), 16 query / 8 KV heads, head_dim 256,
d_model 2560, 262,144-token vocabulary, 64-token pages scattered in the pool.

Prints one JSON line.  `value` is verified tokens per second (tokens the
step emits: accepted drafts plus the target's own token), whole job over
all ranks, timed on the device with CUDA events around each step while the
inputs are resident; `e2e` is the same metric through the C ABI with the
step's inputs copied from pinned host memory and its results copied back
inside the timed region.  `roofline` reports the LM-head kernel (the step's
largest byte mover) against the measured HBM copy bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

Under torchrun each rank runs its own replica of the workload (independent
sequences; no collective on the data path) and rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified tokens/s (k=4) & us per verify step; HBM GB/s as % of B200 peak"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="b1_ctx8k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--draft", action="store_true",
                    help="time the MTP drafter (spec_draft, k steps) on the workload; one JSON line")
    ap.add_argument("--clusters", action="store_true",
                    help="with --draft: the cheap clustered unembedding picks each draft token")
    ap.add_argument("--sweep", action="store_true",
                    help="verify-step time over batch x k on the b1_ctx8k model; one JSON line")
    ap.add_argument("--split-tokens", type=str, default=None,
                    help="tuning: split size of every sliding-window / global layer, 'LOCAL,GLOBAL' "
                         "(recorded in config)")
    ap.add_argument("--profile-case", action="store_true",
                    help="shrink the vocabulary to 4096 (attention and projection shapes kept) "
                         "so that a profiler capture of the layer kernels holds little device "
                         "memory; random drafts; not a benchmark number")
    return ap.parse_args()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def kernel_sources_sha1(files):
    import hashlib
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(key):
    """DRAM bytes (read + write) per launch of a kernel from a committed ncu
    capture, if the sources it was built from are unchanged; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            entry = json.load(f)[key]
        if kernel_sources_sha1(entry["sources"]) != entry["sources_sha1"]:
            return None
        return entry["dram_bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()                      # first sample before timing starts
            while not self.lines and time.time() - t0 < 3.0:
                time.sleep(0.02)
            self.skip = len(self.lines)
        except OSError:
            self.proc = None
            self.skip = 0
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[self.skip:] or self.lines[-1:]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# Inputs: drafts from the workload's recipe; the greedy continuation they
# need comes from the CUDA path itself (k = 0 steps), which only chooses
# inputs and is not a parity claim.
# --------------------------------------------------------------------------

def gpu_greedy_drafts(sess, wl, W):
    import torch
    greedy = np.zeros((wl.batch, wl.k + 1), dtype=np.int64)
    last = np.array([W.last_token(wl, b, sess.attempts[b]) for b in range(wl.batch)], np.int32)
    from speculative_decoding_verification_91_b200.session import WorkloadSession
    g = WorkloadSession(wl.with_(k=0), attempts=sess.attempts, device=sess.device, poison=False)
    cur = last.copy()
    for i in range(wl.k + 1):
        g.set_inputs(cur, [])
        g.step()
        o = g.outputs()
        greedy[:, i] = o["target_ids"][:, 0]
        cur = o["new_last"].astype(np.int32)
    del g
    torch.cuda.empty_cache()
    drafts = np.stack([W.make_drafts(wl, b, sess.attempts[b], greedy[b])[0] for b in range(wl.batch)])
    return last, drafts


def algorithmic_bytes(wl, lens):
    """North-star bytes of one step: visible KV pages read (union of the rows'
    keys; key-equals-value layers at (1+p)*D per token-head) + LM-head weights."""
    kv = 0
    for spec in wl.layers:
        for L in lens:
            hi = L + wl.k + 1
            lo = 0 if spec.window == 0 else max(0, L - spec.window + 1)
            per = (wl.head_dim * (1 + spec.rope_fraction) if spec.kv_equal else 2 * wl.head_dim) * 2
            kv += (hi - lo) * wl.n_kv_heads * per
    lm = wl.vocab * wl.d_model * 2
    proj = sum((wl.qkv_out(s) * wl.d_model + wl.d_model * wl.n_q_heads * wl.head_dim) * 2
               for s in wl.layers)
    return int(kv), int(lm), int(proj)


def launch_labels(wl):
    """Names of the intervals spec_profile_launches reports for one step, in
    launch order (a GEMM and its split-K reduce share one interval)."""
    names = ["embed_norm"]
    for l, spec in enumerate(wl.layers):
        kind = "global" if spec.window == 0 else "local"
        if l > 0:
            names.append(f"L{l}.rmsnorm")
        names += [f"L{l}.qkv_rope", f"L{l}.attn_split[{kind}]", f"L{l}.attn_combine", f"L{l}.o_proj"]
    return names + ["final_rmsnorm", "lm_head_argmax", "accept"]


def attention_bytes(wl, lens, layer):
    spec = wl.layers[layer]
    per = (wl.head_dim * (1 + spec.rope_fraction) if spec.kv_equal else 2 * wl.head_dim) * 2
    kv = 0
    for L in lens:
        hi = L + wl.k + 1
        lo = 0 if spec.window == 0 else max(0, L - spec.window + 1)
        kv += (hi - lo) * wl.n_kv_heads * per
    return int(kv)


def reduce_over_ranks(times, tokens, world, device, launches=0):
    """Whole-job figures of a multi-rank run: every time is the maximum over
    the ranks (the job is as slow as its slowest rank); the emitted tokens and
    the kernel launches of the timed region are summed over the ranks.  One
    all-reduce each; every rank calls it.  Returns (times, tokens, launches)."""
    if world == 1:
        return [float(t) for t in times], int(tokens), int(launches)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in times], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    n = torch.tensor([float(tokens), float(launches)], dtype=torch.float64, device=device)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return [float(v) for v in t.tolist()], int(round(n[0].item())), int(round(n[1].item()))


def run_cuda(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from speculative_decoding_verification_91_b200 import binding as B
    from speculative_decoding_verification_91_b200.inputs import gen
    from speculative_decoding_verification_91_b200.inputs import workloads as W
    from speculative_decoding_verification_91_b200.session import WorkloadSession

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = W.get_workload(args.workload)
    if args.profile_case:
        wl = wl.with_(vocab=4096)
    if args.split_tokens:
        import dataclasses
        loc, glo = (int(x) for x in args.split_tokens.split(","))
        wl = wl.with_(layers=tuple(dataclasses.replace(s, split_tokens=(loc if s.window else glo))
                                   for s in wl.layers))
    B.lib()
    draws = 0
    if args.profile_case:
        sess = WorkloadSession(wl, device=dev, poison=False)
        last = np.array([W.last_token(wl, b, 0) for b in range(wl.batch)], dtype=np.int32)
        drafts = np.stack([gen.randint(wl.seed, f"{wl.name}/profile_drafts", b * wl.k, wl.k, 0, wl.vocab)
                           for b in range(wl.batch)]).astype(np.int32)
        inputs = "profile case: vocabulary 4096, random drafts"
    elif fixture_inputs(wl) is not None:
        # margin-guarded inputs shared with the parity tests; in draws mode
        # every draw has its own context resident and each timed step runs
        # one draw (batch 1), cycling through them
        fx = fixture_inputs(wl)
        sess_wl = wl.with_(batch=len(fx["attempts"])) if fx["draws"] else wl
        sess = WorkloadSession(sess_wl, attempts=fx["attempts"], device=dev, poison=False)
        last, drafts, inputs = fx["last"], fx["drafts"], fx["inputs"]
        draws = len(fx["attempts"]) if fx["draws"] else 0
    else:
        sess = WorkloadSession(wl, device=dev, poison=False)
        last, drafts = gpu_greedy_drafts(sess, wl, W)
        inputs = "attempt-0 draws; drafts from the workload recipe on the CUDA greedy path"
    sess.set_inputs(last, drafts)
    stream = torch.cuda.current_stream(dev)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def one_step(i, with_targets=False):
        if draws:
            sess.step_one(i % draws, stream=stream, with_targets=with_targets)
        else:
            sess.step(stream=stream, with_targets=with_targets)

    # ---- warm-up (untimed), then one untimed pass that fixes the emitted-token
    #      count of every step (of every draw)
    for i in range(args.warmup):
        sess.reset_lengths()
        one_step(i)
    sess.reset_lengths()
    for i in range(max(1, draws)):
        one_step(i, with_targets=True)
    torch.cuda.synchronize(dev)
    out = sess.outputs()
    if sess.ws.device_status(stream) != 0:
        raise RuntimeError("device status flagged during warm-up")
    if draws:
        step_tokens = [int(a) + 1 for a in out["accept_len"]]       # per draw
        if step_tokens != [int(t) for t in fx["draw_tokens"]]:
            raise RuntimeError("emitted tokens differ from the stored oracle outcome")
    else:
        step_tokens = [int(np.sum(out["accept_len"] + 1))]
    tokens_timed = sum(step_tokens[i % len(step_tokens)] for i in range(args.steps))

    # ---- timed: device-resident inputs, L2 flushed before every step; the
    #      library records its own CUDA events around each step and its
    #      LM-head launch on the launching stream
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    B.spec_profile_start(args.steps)
    n_launch0 = B.spec_launch_count()
    torch.cuda.nvtx.range_push("timed")     # selects the timed launches in a profiler
    with ClockSampler(local_rank) as clocks:
        for i in range(args.steps):
            flush.zero_()
            sess.reset_lengths()
            one_step(i)
        torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    n_launches = B.spec_launch_count() - n_launch0
    step_ms, lm_ms = B.spec_profile_collect(args.steps)
    if world > 1:
        dist.barrier()
    if sess.ws.device_status(stream) != 0:
        raise RuntimeError("device status flagged during the timed steps")

    # ---- e2e: the public C-ABI call fed from pinned host buffers (the step's
    #      draw's last token, drafts and length in; its acceptance outputs back)
    Bn, k = wl.batch, wl.k
    n_in = max(1, draws)
    lens_all = sess.lens.astype(np.int32)
    h_in = torch.empty(n_in, Bn * (2 + k), dtype=torch.int32).pin_memory()
    for j in range(n_in):
        sl = slice(j, j + 1) if draws else slice(0, Bn)
        h_in[j, :Bn] = torch.from_numpy(np.ascontiguousarray(last[sl]))
        h_in[j, Bn:Bn + Bn * k] = torch.from_numpy(np.ascontiguousarray(drafts[sl]).reshape(-1).astype(np.int32))
        h_in[j, Bn + Bn * k:] = torch.from_numpy(np.ascontiguousarray(lens_all[sl]))
    h_out = torch.empty(n_in, Bn * (k + 1) + 3 * Bn, dtype=torch.int32).pin_memory()
    e0 = [ev() for _ in range(args.steps)]
    e1 = [ev() for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    q = k + 1
    for i in range(args.steps):
        j = i % n_in
        o = j if draws else 0                         # the draw's slot in the session buffers
        flush.zero_()
        e0[i].record(stream)
        sess.last_token[o:o + Bn].copy_(h_in[j, :Bn], non_blocking=True)
        sess.drafts[o * k:(o + Bn) * k].copy_(h_in[j, Bn:Bn + Bn * k], non_blocking=True)
        sess.seq_lens[o:o + Bn].copy_(h_in[j, Bn + Bn * k:], non_blocking=True)
        one_step(i)
        h_out[j, :Bn * q].copy_(sess.emitted[o * q:(o + Bn) * q], non_blocking=True)
        h_out[j, Bn * q:Bn * (q + 1)].copy_(sess.accept_len[o:o + Bn], non_blocking=True)
        h_out[j, Bn * (q + 1):Bn * (q + 2)].copy_(sess.new_last[o:o + Bn], non_blocking=True)
        h_out[j, Bn * (q + 2):].copy_(sess.seq_lens[o:o + Bn], non_blocking=True)
        e1[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = [s.elapsed_time(e) for s, e in zip(e0, e1)]
    for j in range(min(n_in, args.steps)):
        got_acc = h_out[j, Bn * q:Bn * (q + 1)].numpy()
        want = out["accept_len"][j:j + 1] if draws else out["accept_len"]
        assert np.array_equal(got_acc, want), "e2e step disagrees with the device-timed step"

    # per-launch breakdown of one extra step (events serialise the launches)
    flush.zero_()
    sess.reset_lengths()
    B.spec_profile_launches(256)
    one_step(0)
    launch_ms = B.spec_profile_launches_collect(256)

    mean_step = float(np.mean(step_ms))
    mean_lm = float(np.mean(lm_ms))
    mean_e2e = float(np.mean(e2e_ms))
    (mean_step, mean_e2e, mean_lm), tokens_all, n_launches = reduce_over_ranks(
        [mean_step, mean_e2e, mean_lm], tokens_timed, world, dev, n_launches)
    lens = sess.lens[:1] if draws else sess.lens
    kv_b, lm_b, proj_b = algorithmic_bytes(wl, lens)
    tps = fx["tokens_per_step"] if draws else tokens_timed / args.steps
    return dict(wl=wl, lens=lens, tokens_per_step=tps, tokens_all=tokens_all,
                mean_step=mean_step, inputs=inputs, draws=draws,
                mean_lm=mean_lm, mean_e2e=mean_e2e, kv_b=kv_b, lm_b=lm_b, proj_b=proj_b,
                launches=n_launches, clocks=clocks.summary(),
                h2d=int(h_in[0].numel() * 4), d2h=int(h_out[0].numel() * 4), step_ms=step_ms,
                M=wl.batch * wl.q_rows, launch_us=[round(x * 1e3, 1) for x in launch_ms])


# --------------------------------------------------------------------------
# CPU oracle leg (baseline only; bounded sample)
# --------------------------------------------------------------------------

def fixture_inputs(wl):
    """The margin-guarded step inputs stored for the workload (written by the
    oracle-only script beside them), or None: per-sequence draw attempts, last
    tokens, drafts, the emitted-token count of the step and a description."""
    fixture = os.path.join(ROOT, "tests", "golden", f"verify_{wl.name}.json")
    if not os.path.exists(fixture):
        return None
    with open(fixture) as f:
        seqs = json.load(f)["sequences"]
    with open(fixture) as f:
        draws = json.load(f).get("mode") == "draws"
    toks = [q["accept_len"] + 1 for q in seqs]
    inputs = "margin-guarded fixture " + os.path.relpath(fixture, ROOT)
    if draws:
        inputs += (f"; {len(seqs)} draws cycled one per step (batch 1 each), mean emitted tokens "
                   f"per step {np.mean(toks):.4f}")
    return dict(attempts=[q["attempt"] for q in seqs],
                last=np.array([q["last_token"] for q in seqs], dtype=np.int32),
                drafts=np.array([q["drafts"] for q in seqs], dtype=np.int32),
                draws=draws, draw_tokens=toks,
                # draws: mean emitted tokens of one batch-1 step; else of the batched step
                tokens_per_step=round(float(np.mean(toks)), 4) if draws else int(sum(toks)),
                inputs=inputs)


def workload_config(wl, lens, tokens_per_step, inputs):
    """The JSON line's `config`, the same object for both arms."""
    return {"workload": wl.name, "batch": wl.batch, "k": wl.k,
            "split_tokens": [s.split_tokens or wl.split_tokens for s in wl.layers],
            "context": [int(x) for x in lens], "layers": len(wl.layers),
            "d_model": wl.d_model, "vocab": wl.vocab,
            "l2": f"flushed ({L2_FLUSH_BYTES >> 20} MiB write) before every timed step",
            "tokens_per_step": tokens_per_step, "inputs": inputs}


def oracle_setup(wl_name: str):
    """The oracle's model, caches and inputs for sequence 0 of the workload
    (the stored margin-guarded inputs when the workload has them, as in the
    CUDA arm)."""
    import oracle
    from speculative_decoding_verification_91_b200.inputs import workloads as W
    from speculative_decoding_verification_91_b200.inputs import gen
    wl = W.get_workload(wl_name)
    L = int(W.context_lengths(wl)[0])
    fx = fixture_inputs(wl)
    attempt = fx["attempts"][0] if fx else 0
    layers = []
    for l, spec in enumerate(wl.layers):
        wqkv, wo = W.layer_weights(wl, l)
        layers.append(oracle.LayerDef(spec.window, spec.kv_equal, spec.rope_fraction,
                                      oracle.bf16_from_bits(wqkv), oracle.bf16_from_bits(wo)))
    model = oracle.Model(wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                         W.lm_head_weight(wl), layers, wl.rope_theta, wl.rms_eps,
                         W.embedding_weight(wl))
    caches = []
    for l in range(len(wl.layers)):
        lo, k, v = W.context_kv(wl, 0, attempt, l, L)
        caches.append(oracle.cache_from_raw(model, l, lo, oracle.bf16_from_bits(k),
                                            None if v is None else oracle.bf16_from_bits(v)))
    if fx:
        last, drafts = int(fx["last"][0]), fx["drafts"][0]
    else:
        last = W.last_token(wl, 0, 0)
        drafts = gen.randint(wl.seed, f"{wl.name}/bench_drafts", 0, wl.k, 0, wl.vocab)
    return wl, model, caches, L, last, drafts


def run_reference(args):
    """--impl reference: the oracle (numpy float64) on the host cores, timed as
    K steps after W warm-up steps within about two minutes.  Calibration: one
    full oracle verify step of sequence 0, split into its layer stack (embed,
    layers, final norm) and its LM head.  Each step then re-times the LM head
    on a vocabulary slice sized to the step's share of the time budget and
    estimates the step as layer time + slice time scaled to the whole
    vocabulary; the metric is emitted tokens / estimated step time."""
    import oracle
    wl, model, caches, L, last, drafts = oracle_setup(args.workload)
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    toks = [int(last)] + [int(t) for t in drafts]
    t0 = time.perf_counter()
    fw = oracle.verify_forward(model, caches, L, toks, lm_rows=[])
    h = oracle.bf16(oracle.rmsnorm(fw.x_out, model.rms_eps))     # every row's final hidden state
    t_layers = time.perf_counter() - t0
    t0 = time.perf_counter()
    g, _, _ = oracle.lm_head_top2(h, model.w_lm_bits)
    t_lm = time.perf_counter() - t0
    a, _, _ = oracle.accept_longest_prefix([int(t) for t in drafts], g)
    fx = fixture_inputs(wl)
    # draws mode: the stored draws' mean emitted tokens (each draw's step costs the same)
    tokens_per_step = fx["tokens_per_step"] if fx and fx["draws"] else a + 1
    V = model.vocab
    budget = max(0.005, 120.0 / max(1, args.steps + args.warmup))
    n_slice = int(min(V, max(1024, V * budget / max(t_lm, 1e-9))))
    est = []
    for i in range(args.warmup + args.steps):
        v0 = (i * n_slice) % max(1, V - n_slice + 1)
        t0 = time.perf_counter()
        oracle.lm_head_top2(h, model.w_lm_bits[v0:v0 + n_slice])
        ts = time.perf_counter() - t0
        est.append(t_layers + ts * V / n_slice)
    sec = float(np.mean(est[args.warmup:]))
    tps = tokens_per_step / sec
    desc = (f"oracle on sequence 0 of {wl.name} ({len(wl.layers)} layers, k={wl.k}, ctx {L}, vocab {V}); "
            f"layer stack timed once ({t_layers:.2f} s), each step times the LM head on {n_slice} "
            f"of {V} tokens and scales it to the vocabulary; numpy float64, BLAS threads={threads}")
    if wl.batch > 1:
        desc += f"; the metric is sequence 0's emitted tokens over its step time (batch {wl.batch})"
    from speculative_decoding_verification_91_b200.inputs import workloads as W
    fx = fixture_inputs(wl)
    config = workload_config(wl, W.context_lengths(wl), fx["tokens_per_step"] if fx else tokens_per_step,
                             fx["inputs"] if fx else "attempt-0 draws; random drafts")
    return tps, sec, threads, desc, config


def oracle_sample(wl_name: str, budget_s: float = 25.0):
    """Times the CPU oracle on one sequence of the workload: a full verify
    step (all layers, all k+1 rows, full-vocabulary LM head).  Returns
    (tokens/s, seconds, threads, description)."""
    import oracle
    wl, model, caches, L, last, drafts = oracle_setup(wl_name)
    t0 = time.perf_counter()
    n = 0
    tokens = 0
    while True:
        res = oracle.verify_step(model, caches, L, last, drafts)
        tokens += res.accept_len + 1
        n += 1
        if time.perf_counter() - t0 > budget_s * 0.5 or n >= 3:
            break
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = (f"{n} full oracle verify step(s) of sequence 0 ({wl.name}: {len(wl.layers)} layers, "
            f"k={wl.k}, ctx {L}, vocab {wl.vocab}); numpy float64, BLAS threads={threads}")
    return tokens / dt, dt / n, threads, desc


def run_lmhead_only(args):
    """--workload lmhead:M,d,V: the LM head + argmax kernel alone on random bf16
    inputs, L2 flushed before every launch; reports its roofline."""
    import torch
    from speculative_decoding_verification_91_b200 import binding as B
    from speculative_decoding_verification_91_b200.inputs import gen
    from speculative_decoding_verification_91_b200.runtime import Workspace, to_device_bf16
    M, d, V = (int(x) for x in args.workload.split(":")[1].split(","))
    torch.cuda.set_device(0)
    h = to_device_bf16(gen.normal_bf16(0, "bench/lm/h", 0, M * d, 1.0), "cuda")
    w = to_device_bf16(gen.normal_bf16(0, "bench/lm/w", 0, V * d, 0.02), "cuda")
    ws = Workspace(B.spec_lmhead_workspace_bytes(M, V))
    ids = torch.zeros(M, dtype=torch.int32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        B.spec_lmhead_argmax(h, w, M, d, V, ids, None, ws.buf, ws.nbytes)
    t0 = [ev() for _ in range(args.steps)]
    t1 = [ev() for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        t0[i].record()
        B.spec_lmhead_argmax(h, w, M, d, V, ids, None, ws.buf, ws.nbytes)
        t1[i].record()
    torch.cuda.synchronize()
    us = float(np.mean([a.elapsed_time(b) for a, b in zip(t0, t1)])) * 1e3
    byts = V * d * 2 + M * d * 2
    flops = 2.0 * M * d * V
    peak, kind = measured_peaks()
    tf = None
    mp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(mp):
        tf = json.load(open(mp)).get("bf16_tflops")
    print(json.dumps({"kernel": "lmhead_argmax", "M": M, "d": d, "V": V, "us": us,
                      "gbs": byts / us / 1e3, "frac_hbm": byts / us / 1e3 / peak,
                      "tflops": flops / us / 1e6,
                      "frac_tensor": (flops / us / 1e6 / tf) if tf else None}), flush=True)


def lm_roofline(wl, r, lm_bytes, lm_s, peak_gbs, peak_kind):
    """Roofline of the step's dominant kernel, the LM head + argmax.  Its
    bound is the larger of bytes / measured copy bandwidth and FLOPs /
    measured sustained bf16 GEMM throughput (it runs inside a long step):
    HBM for few verify rows, the tensor cores at 256 rows."""
    M = r["M"]
    flops = 2.0 * M * wl.d_model * wl.vocab
    tf = None
    mp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(mp):
        tf = json.load(open(mp)).get("bf16_tflops_sustained")
    kernel = ("tc_gemm_kernel<argmax> (tcgen05 LM head + argmax)" if 32 < M <= 256
              else "stream_gemm_kernel<argmax> (LM head + argmax + acceptance)")
    t_hbm = lm_bytes / (peak_gbs * 1e9)
    t_tc = flops / (tf * 1e12) if tf else 0.0
    out = {"kernel": kernel, "bytes_per_launch": lm_bytes, "flops_per_launch": flops,
           "us_per_launch": lm_s * 1e6,
           "traffic": measured_traffic(f"lm_head_argmax/{wl.name}")}
    if t_tc > t_hbm:
        ach = flops / lm_s / 1e12
        out.update({"bound": "tensor", "achieved": ach, "peak": tf, "unit": "TFLOP/s",
                    "frac": ach / tf, "peak_kind": "measured sustained bf16 GEMM"})
    else:
        ach = lm_bytes / lm_s / 1e9
        out.update({"bound": "hbm", "achieved": ach, "peak": peak_gbs, "unit": "GB/s",
                    "frac": ach / peak_gbs, "peak_kind": peak_kind})
    return out


def attention_roofline(wl, r, peak):
    """Per layer: visible KV bytes / (split + combine interval) of the
    per-launch breakdown (launches serialised by events there, so slightly
    pessimistic)."""
    labels = launch_labels(wl)
    if len(labels) != len(r["launch_us"]):
        return None
    us = dict(zip(labels, r["launch_us"]))
    out = []
    for l, spec in enumerate(wl.layers):
        t = [v for k, v in us.items() if k.startswith(f"L{l}.attn_split")][0] + us[f"L{l}.attn_combine"]
        b = attention_bytes(wl, r["lens"], l)
        out.append({"layer": l, "kind": "global" if spec.window == 0 else "local", "bytes": b,
                    "us": t, "gbs": b / t / 1e3, "frac_of_measured": b / t / 1e3 / peak})
    return out


SWEEP_B = (1, 2, 4, 8, 16, 32, 64)
SWEEP_K = (0, 1, 2, 4, 8, 16)


def expected_tokens(alpha, k):
    """Emitted tokens per verify step when every draft is right with
    probability alpha independently: sum_{i=0..k} alpha^i."""
    return sum(alpha ** i for i in range(k + 1))


def run_sweep(args):
    """--sweep: the fused verify step over batch sizes B and draft counts k on
    the b1_ctx8k model (2 layers, d_model 2560, vocab 262,144, every sequence
    at context 8192).  One session sized for the largest B and k; smaller
    configurations use its first B sequences.  The cache pages are zero (the
    step time does not depend on their values); L2 is flushed before every
    timed step.  Reports us per step, its ratio to the k = 0 step (a plain
    decode step through the same kernels) and the speed-up over decoding
    that i.i.d. acceptance alpha = 0.8 would give."""
    import torch
    from speculative_decoding_verification_91_b200 import binding as B
    from speculative_decoding_verification_91_b200.inputs import workloads as W
    from speculative_decoding_verification_91_b200.session import WorkloadSession
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = W.get_workload("b1_ctx8k").with_(name="sweep", batch=max(SWEEP_B), k=max(SWEEP_K))
    sess = WorkloadSession(wl, device=dev, poison=False, fill_context=False)
    for pools in (sess.dm.k_pool, sess.dm.v_pool, sess.dm.ksb_pool):
        for p in pools:
            if p is not None:
                p.zero_()
    sess.set_inputs(np.zeros(wl.batch, np.int32), np.ones((wl.batch, wl.k), np.int32))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    d = sess.dm.desc

    def step(Bn, k):
        B.spec_verify_step(d, sess.block_table, sess.max_pages, sess.last_token,
                           sess.drafts if k > 0 else None, Bn, k, sess.seq_lens, sess.accept_len,
                           sess.emitted, sess.new_last, None, None, sess.ws.buf, sess.ws.nbytes, stream)

    steps = max(3, min(args.steps, 50))
    out = []
    with ClockSampler(0) as clocks:
        for Bn in SWEEP_B:
            t0 = None
            for k in SWEEP_K:
                for _ in range(max(3, args.warmup)):
                    sess.reset_lengths()
                    step(Bn, k)
                torch.cuda.synchronize(dev)
                B.spec_profile_start(steps)
                for _ in range(steps):
                    flush.zero_()
                    sess.reset_lengths()
                    step(Bn, k)
                torch.cuda.synchronize(dev)
                ms, _ = B.spec_profile_collect(steps)
                us = float(np.mean(ms)) * 1e3
                t0 = us if k == 0 else t0
                ratio = us / t0
                out.append({"B": Bn, "k": k, "rows": Bn * (k + 1), "us_per_step": round(us, 1),
                            "vs_k0": round(ratio, 3),
                            "speedup_at_alpha_0.8": round(expected_tokens(0.8, k) / ratio, 3)})
    if sess.ws.device_status(stream) != 0:
        raise RuntimeError("device status flagged during the sweep")
    print(json.dumps({"sweep": "verify step, batch x k", "workload": "b1_ctx8k model, context 8192",
                      "steps_per_point": steps, "l2": "flushed before every timed step",
                      "points": out, "clocks": clocks.summary()}), flush=True)


def run_draft_bench(args):
    """--draft: k drafter steps (spec_draft) for the workload's batch on its
    target cache: 4 blocks (3 sliding-window, 1 global) of width 256, each
    step ending in the target's LM head over the full vocabulary.  Inputs
    resident; L2 flushed before every timed call; CUDA events on the stream."""
    import torch
    from speculative_decoding_verification_91_b200 import binding as B
    from speculative_decoding_verification_91_b200.inputs import workloads as W
    from speculative_decoding_verification_91_b200.runtime import (DeviceClusters, DeviceDrafter,
                                                                    Workspace, to_device_bf16)
    from speculative_decoding_verification_91_b200.session import WorkloadSession
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = W.get_workload(args.workload)
    sess = WorkloadSession(wl, device=dev, poison=False)
    dd, hq, targets = W.drafter_spec(wl)
    emb, down, upw, blocks = W.drafter_weights(wl)
    cl = None
    if args.clusters:
        cl_tokens, cent, wc, n_sel = W.cluster_tables(wl)
        cl = DeviceClusters(cluster_tokens=cl_tokens, centroid_bits=cent, clustered_bits=wc,
                            n_select=n_sel, device=dev)
    dr = DeviceDrafter(d_draft=dd, n_q_heads=hq, w_emb_bits=emb, w_down_bits=down, w_up_bits=upw,
                       blocks=blocks, device=dev, clusters=cl)
    Bn, k = wl.batch, max(1, wl.k)
    hidden = to_device_bf16(np.stack([W.drafter_inputs(wl, b, 0)[0] for b in range(Bn)]), dev)
    toks = torch.tensor([W.drafter_inputs(wl, b, 0)[1] for b in range(Bn)], dtype=torch.int32, device=dev)
    ws = Workspace(B.spec_draft_workspace_bytes(sess.dm.desc, dr.desc, Bn, sess.max_pages), dev)
    drafts = torch.zeros(Bn * k, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        B.spec_draft(sess.dm.desc, dr.desc, sess.block_table, sess.max_pages, sess.seq_lens, hidden,
                     toks, Bn, k, drafts, None, ws.buf, ws.nbytes, stream)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, 200))
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    n0 = B.spec_launch_count()
    with ClockSampler(0) as clocks:
        for i in range(steps):
            flush.zero_()
            e0[i].record(stream)
            call()
            e1[i].record(stream)
        torch.cuda.synchronize(dev)
    launches = B.spec_launch_count() - n0
    if ws.device_status(stream) != 0:
        raise RuntimeError("device status flagged during the drafter calls")
    us = float(np.mean([a.elapsed_time(b) for a, b in zip(e0, e1)])) * 1e3
    lm_bytes = wl.vocab * wl.d_model * 2
    unembed = None
    if cl is not None:
        # the unembedding alone: clusters vs the full LM head, same rows
        hrows = torch.randn(Bn, wl.d_model, device=dev).to(torch.bfloat16)
        ids = torch.zeros(Bn, dtype=torch.int32, device=dev)
        wsc = Workspace(B.spec_cluster_unembed_workspace_bytes(Bn, wl.d_model, cl.desc), dev)
        wsl = Workspace(B.spec_lmhead_workspace_bytes(Bn, wl.vocab), dev)
        def t_of(fn, n=50):
            for _ in range(3):
                fn()
            a = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            z = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            for i in range(n):
                flush.zero_()
                a[i].record(stream)
                fn()
                z[i].record(stream)
            torch.cuda.synchronize(dev)
            return float(np.mean([x.elapsed_time(y) for x, y in zip(a, z)])) * 1e3
        t_cl = t_of(lambda: B.spec_cluster_unembed(hrows, Bn, wl.d_model, cl.desc, ids, None, wsc.buf,
                                                    wsc.nbytes, stream))
        t_lm = t_of(lambda: B.spec_lmhead_argmax(hrows, sess.dm.w_lm, Bn, wl.d_model, wl.vocab, ids,
                                                  None, wsl.buf, wsl.nbytes, stream))
        C, S = cl_tokens.shape
        cand_bytes = Bn * n_sel * S * wl.d_model * 2 + C * wl.d_model * 2
        unembed = {"clusters": C, "cluster_size": S, "n_select": n_sel,
                   "us_cluster_unembed": t_cl, "us_full_lm_head": t_lm,
                   "bytes_cluster_unembed": cand_bytes, "bytes_full_lm_head": lm_bytes}
    print(json.dumps({"kernel": "spec_draft", "workload": wl.name, "batch": Bn, "k": k,
                      "unembed": "clusters" if cl is not None else "full LM head",
                      "unembed_alone": unembed,
                      "d_draft": dd, "blocks_target_layers": targets,
                      "us_per_call": us, "us_per_draft_step": us / k,
                      "drafted_tokens_per_s": Bn * k / (us / 1e6),
                      "lm_head_bytes_per_step": lm_bytes,
                      "gpu_launches_per_call": launches / steps,
                      "l2": "flushed before every timed call", "clocks": clocks.summary()}), flush=True)


def loop_drafter(wl, greedy_stream):
    """The loop workload's corrupted-greedy drafter: draft i of a step is the
    true greedy token (from the precomputed greedy stream, at the sequence's
    emitted position) with probability p, else a random id (seeded flips)."""
    def drafter(step, n_emitted):
        flips, ids = W_mod().loop_draft_flips(wl, step)
        out = []
        for i in range(wl.k):
            e = n_emitted + i
            truth = greedy_stream[e] if e < len(greedy_stream) else 0
            out.append(truth if flips[i] < wl.accept[1] else int(ids[i]))
        return np.asarray(out, dtype=np.int32)
    return drafter


def W_mod():
    from speculative_decoding_verification_91_b200.inputs import workloads as W
    return W


def run_loop(args):
    """--workload loop_131k: the speculative loop after a 131,072-token prompt.

    Untimed: the prompt is prefilled on the GPU (spec_prefill, 256-token
    chunks) and the greedy stream the drafter corrupts is produced by k = 0
    steps; then the lengths are rolled back to the prompt.  Timed: the loop's
    verify steps (min(--steps, 512)), each with drafts built on the host from
    the tokens emitted so far; L2 flushed before every step.  Per step the
    library's CUDA events give the device time of spec_verify_step; the e2e
    figure adds the host->device copy of the step's inputs (last token,
    drafts) and the device->host copy of its outputs, which the loop needs
    anyway to build the next drafts.  --warmup steps run first and are rolled
    back (rollback = resetting the length)."""
    import torch
    from speculative_decoding_verification_91_b200 import binding as B
    from speculative_decoding_verification_91_b200.session import WorkloadSession
    W = W_mod()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = W.get_workload(args.workload)
    steps = max(1, min(args.steps, wl.steps))
    s = WorkloadSession(wl, fill_context=False, lens=np.zeros(wl.batch, np.int64), device=dev,
                        poison=False, extra_tokens=wl.prompt_tokens + (steps + args.warmup + 2) * (wl.k + 1))
    t0 = time.time()
    nxt, _ = s.prefill(W.prompt_tokens(wl)[None, :])
    t_prefill = time.time() - t0
    L0 = int(s.seq_lens[0].item())
    n_greedy = steps * (wl.k + 1) + 1
    greedy, _ = s.greedy(nxt, n_greedy)
    stream_tokens = [int(t) for t in greedy[0]]
    drafter = loop_drafter(wl, stream_tokens)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    k, q = wl.k, wl.k + 1
    h_in = torch.empty(1 + k, dtype=torch.int32).pin_memory()
    h_out = torch.empty(q + 3, dtype=torch.int32).pin_memory()

    def run(n, timed):
        s.seq_lens.fill_(L0)
        cur, emitted, accepts = int(nxt[0]), 0, []
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        if timed:
            B.spec_profile_start(n)
            torch.cuda.nvtx.range_push("timed")
        for st in range(n):
            h_in[0] = cur
            h_in[1:] = torch.from_numpy(drafter(st, emitted))
            flush.zero_()
            e0[st].record(stream)
            s.last_token.copy_(h_in[:1], non_blocking=True)
            s.drafts[:k].copy_(h_in[1:], non_blocking=True)
            s.step(stream=stream, with_targets=False)
            h_out[:q].copy_(s.emitted[:q], non_blocking=True)
            h_out[q:q + 1].copy_(s.accept_len[:1], non_blocking=True)
            h_out[q + 1:q + 2].copy_(s.new_last[:1], non_blocking=True)
            h_out[q + 2:].copy_(s.seq_lens[:1], non_blocking=True)
            e1[st].record(stream)
            stream.synchronize()               # the drafter needs this step's tokens
            a = int(h_out[q])
            got = [int(x) for x in h_out[:a + 1]]
            if got != stream_tokens[emitted:emitted + a + 1]:
                raise RuntimeError(f"loop step {st} emitted tokens that differ from greedy decoding")
            accepts.append(a)
            emitted += a + 1
            cur = int(h_out[q + 1])
        torch.cuda.synchronize(dev)
        if timed:
            torch.cuda.nvtx.range_pop()
        e2e = [x.elapsed_time(y) for x, y in zip(e0, e1)]
        dev_ms = B.spec_profile_collect(n)[0] if timed else None
        return accepts, dev_ms, e2e

    if args.warmup:
        run(args.warmup, False)
    # per-launch breakdown of one verify step at the prompt's end (events
    # serialise the launches; rolled back afterwards)
    s.seq_lens.fill_(L0)
    s.last_token.fill_(int(nxt[0]))
    s.drafts[:k].copy_(torch.from_numpy(drafter(0, 0)))
    flush.zero_()
    B.spec_profile_launches(256)
    s.step(stream=stream, with_targets=False)
    launch_ms = B.spec_profile_launches_collect(256)
    labels = launch_labels(wl)
    breakdown = (dict(zip(labels, [round(x * 1e3, 1) for x in launch_ms])) if len(labels) == len(launch_ms)
                 else [round(x * 1e3, 1) for x in launch_ms])
    n0 = B.spec_launch_count()
    with ClockSampler(0) as clocks:
        accepts, dev_ms, e2e = run(steps, True)
    launches = B.spec_launch_count() - n0
    if s.ws.device_status(stream) != 0:
        raise RuntimeError("device status flagged during the loop")
    tokens = int(sum(a + 1 for a in accepts))
    total_s = float(np.sum(dev_ms)) / 1e3
    e2e_s = float(np.sum(e2e)) / 1e3
    # bytes of each step at its own committed length
    lens, L = [], L0
    for a in accepts:
        lens.append(L)
        L += a + 1
    kv = [algorithmic_bytes(wl, [x])[0] for x in lens]
    _, lm_b, proj_b = algorithmic_bytes(wl, [L0])
    step_bytes = float(np.mean(kv)) + lm_b
    mean_step = total_s / steps
    peak, peak_kind = measured_peaks()
    value = tokens / total_s
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": steps,
            "warmup": args.warmup, "ms_per_step": mean_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "k": wl.k,
                       "prompt": wl.prompt_tokens, "loop_steps": steps,
                       "context": [L0, L], "layers": len(wl.layers), "d_model": wl.d_model,
                       "vocab": wl.vocab, "l2": f"flushed ({L2_FLUSH_BYTES >> 20} MiB write) before every step",
                       "tokens_per_step": tokens / steps,
                       "inputs": "131,072 random prompt tokens prefilled on the GPU (untimed); "
                                 "corrupted-greedy drafts (p = 0.8) built on the host each step; "
                                 "every step's emitted tokens checked against greedy decoding"},
            "us_per_step": mean_step * 1e6,
            "step_hbm": {"bytes": step_bytes, "bytes_with_projections": step_bytes + proj_b,
                         "gbs": step_bytes / mean_step / 1e9,
                         "frac_of_8tbs": step_bytes / mean_step / 1e9 / NOMINAL_HBM_GBS,
                         "frac_of_measured": step_bytes / mean_step / 1e9 / peak},
            "accept_len_mean": float(np.mean(accepts)),
            "e2e": {"value": tokens / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": int(h_in.numel() * 4),
                    "d2h_bytes_per_step": int(h_out.numel() * 4)},
            "gpu_launches": launches, "launch_breakdown_us": breakdown,
            "prefill_s": round(t_prefill, 2), "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.workload == "loop_131k" and args.impl == "cuda":
        run_loop(args)
        return
    if args.draft:
        run_draft_bench(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.workload.startswith("lmhead:"):
        run_lmhead_only(args)
        return
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        if rank != 0:
            return
        tps, sec, threads, desc, config = run_reference(args)
        line = {"metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": config,
                "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": threads,
                                 "kind": "oracle", "sample": desc},
                "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=300))
    try:
        r = run_cuda(args, rank, world, local_rank)
    finally:
        pass
    if rank == 0:
        wl = r["wl"]
        peak, peak_kind = measured_peaks()
        step_s = r["mean_step"] / 1e3
        lm_s = r["mean_lm"] / 1e3
        # whole job: tokens emitted over the timed steps (all ranks) / their time
        value = r["tokens_all"] / (args.steps * step_s)
        lm_bytes = r["lm_b"] + r["M"] * wl.d_model * 2
        step_bytes = r["kv_b"] + r["lm_b"]
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["mean_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(wl, r["lens"], r["tokens_per_step"], r["inputs"]),
            "us_per_step": r["mean_step"] * 1e3,
            "step_hbm": {"bytes": step_bytes, "bytes_with_projections": step_bytes + r["proj_b"],
                         "gbs": step_bytes / step_s / 1e9,
                         "frac_of_8tbs": step_bytes / step_s / 1e9 / NOMINAL_HBM_GBS,
                         "frac_of_measured": step_bytes / step_s / 1e9 / peak},
            "roofline": lm_roofline(wl, r, lm_bytes, lm_s, peak, peak_kind),
            "e2e": {"value": r["tokens_all"] / (args.steps * r["mean_e2e"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
            "gpu_launches": r["launches"],
            "launch_breakdown_us": dict(zip(launch_labels(wl), r["launch_us"]))
            if len(launch_labels(wl)) == len(r["launch_us"]) else r["launch_us"],
            "attention_hbm": attention_roofline(wl, r, peak),
            "clocks": r["clocks"],
        }
        if not args.no_cpu_baseline and world == 1:
            _, sec, threads, desc = oracle_sample(wl.name)
            line["cpu_baseline"] = {"value": r["tokens_per_step"] / sec, "unit": "tokens/s",
                                    "cores": threads, "kind": "oracle",
                                    "sample": desc + f"; s/step {sec:.2f}, scaled by the "
                                    f"workload's {r['tokens_per_step']} emitted tokens per step"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
