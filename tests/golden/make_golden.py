"""Writes tests/golden/verify_<workload>.json: margin-guarded inputs and the
oracle's expected outcome of one verify step at the workload's full size.

Calls only the oracle and the seeded input generator.  For every sequence
the sub-seed (context, last token, drafts) is redrawn (attempt 0, 1, ...)
until every argmax the acceptance depends on (rows 0..a) has a top-2 gap
above the logits' float tolerance (2e-2 + 1e-2*|top1|), so any
implementation within that tolerance takes the same decisions.

LM-head passes are batched over all sequences of a round so that the
262,144-row vocabulary is streamed once per round, not once per row.

Draws mode (`name:draws=N`): N independent single-sequence steps of the
workload, draw b seeded as sequence b of its seed space.  Each draw's
rejection point is taken once from the recipe (attempt 0's coin flips) and
kept while its context and last token are redrawn for the margin guard, so
the stored draws follow the recipe's acceptance distribution (a guard that
also redrew the rejection point would favour short accepted runs, which
have fewer rows to guard).

  python tests/golden/make_golden.py b1_ctx8k:draws=24 [b8_ragged ...]
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from speculative_decoding_verification_91_b200.inputs import workloads as W  # noqa: E402
from tests import harness  # noqa: E402


def _forward_rows(model, caches, L, tokens):
    fw = oracle.verify_forward(model, caches, L, tokens, lm_rows=[])
    return fw


def solve(wl: W.Workload, max_rounds: int = 60, log=print, fixed_r: bool = False):
    model = harness.oracle_model(wl)
    lens = W.context_lengths(wl)
    attempt = [0] * wl.batch
    done = {}
    t0 = time.time()
    for rnd in range(max_rounds):
        todo = [b for b in range(wl.batch) if b not in done]
        if not todo:
            break
        state = {}
        for b in todo:
            L = int(lens[b])
            caches = harness.context_caches(wl, model, b, attempt[b], L)
            last = W.last_token(wl, b, attempt[b])
            r = W.rejection_point(wl, b, 0 if fixed_r else attempt[b])
            need = wl.k if (r == wl.k or wl.accept[0] == "one_wrong") else r + 1
            state[b] = dict(L=L, caches=caches, last=last, r=r, need=need, greedy=[])
        # greedy continuation, one batched LM pass per position
        for j in range(wl.k + 1):
            rows, owners = [], []
            for b in todo:
                st = state[b]
                if len(st["greedy"]) < st["need"] and len(st["greedy"]) == j:
                    fw = _forward_rows(model, st["caches"], st["L"], [st["last"]] + st["greedy"])
                    rows.append(oracle.bf16(oracle.rmsnorm(fw.x_out[-1:], model.rms_eps)))
                    owners.append(b)
            if not rows:
                break
            ids, _, _ = oracle.lm_head_top2(np.concatenate(rows), model.w_lm_bits)
            for b, g in zip(owners, ids):
                state[b]["greedy"].append(int(g))
        # the verify step itself, one batched LM pass for all rows
        rows, spans = [], []
        for b in todo:
            st = state[b]
            drafts, r2 = W.make_drafts(wl, b, attempt[b], np.array(st["greedy"] + [0], np.int64),
                                       r=st["r"])
            st["drafts"] = drafts
            fw = _forward_rows(model, st["caches"], st["L"], [st["last"]] + [int(x) for x in drafts])
            h = oracle.bf16(oracle.rmsnorm(fw.x_out, model.rms_eps))
            spans.append((b, len(rows), h.shape[0]))
            rows.extend(list(h))
        ids, t1, t2 = oracle.lm_head_top2(np.stack(rows), model.w_lm_bits)
        for b, s0, n in spans:
            st = state[b]
            g, a1, a2 = ids[s0:s0 + n], t1[s0:s0 + n], t2[s0:s0 + n]
            a, emitted, nxt = oracle.accept_longest_prefix(st["drafts"], g)
            ok = a == st["r"] and all(harness.margin_ok(a1[i], a2[i]) for i in range(a + 1))
            if ok:
                done[b] = dict(b=b, attempt=attempt[b], L=st["L"], last_token=st["last"],
                               drafts=[int(x) for x in st["drafts"]], r=st["r"], accept_len=a,
                               emitted=emitted, next_last_token=nxt, new_len=st["L"] + a + 1,
                               target_ids=[int(x) for x in g], top1=[float(x) for x in a1],
                               top2=[float(x) for x in a2],
                               margin_ok=[bool(harness.margin_ok(a1[i], a2[i])) for i in range(n)])
            else:
                attempt[b] += 1
        log(f"[{wl.name}] round {rnd}: {len(done)}/{wl.batch} sequences guarded "
            f"({time.time() - t0:.0f}s)")
    if len(done) != wl.batch:
        raise RuntimeError(f"{wl.name}: {wl.batch - len(done)} sequences without a safe draw")
    return [done[b] for b in range(wl.batch)]


def main(names):
    for arg in names:
        name, _, opt = arg.partition(":")
        wl = W.get_workload(name)
        draws = int(opt.split("=")[1]) if opt.startswith("draws=") else 0
        if draws:
            seqs = solve(wl.with_(batch=draws), fixed_r=True)
        else:
            seqs = solve(wl)
        out = {
            "_about": ("Margin-guarded inputs and the oracle's outcome of one verify step; "
                       "written by tests/golden/make_golden.py (oracle + seeded inputs only)."),
            "workload": name,
            "margin": {"abs": harness.MARGIN_ABS, "rel": harness.MARGIN_REL},
            "sequences": seqs,
        }
        if draws:
            out["mode"] = "draws"
            out["_about"] += (f" Draws mode: {draws} independent batch-1 steps (draw b = sequence b "
                              "of the seed space); rejection points fixed per draw from the "
                              "recipe, contexts redrawn for the margin guard.")
        path = os.path.join(HERE, f"verify_{name}.json")
        with open(path, "w") as f:
            json.dump(out, f, indent=1)
        print(f"wrote {path}")


if __name__ == "__main__":
    main(sys.argv[1:] or ["b1_ctx8k"])
