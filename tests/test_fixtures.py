"""The stored margin-guarded fixtures (`tests/golden/verify_*.json`, written
by `tests/golden/make_golden.py` from the oracle) against the draft recipe
and the acceptance rule, on CPU:

* every stored rejection point is the recipe's (attempt 0's coin flips for
  the b1_ctx8k draws, which keep it fixed while the margin guard redraws the
  context; the stored attempt's otherwise), and the stored drafts are the
  recipe's drafts for it;
* the stored outcome follows from the stored target ids by the acceptance
  rule: a = leading drafts equal to the target's argmax (the recipe makes it
  the rejection point), the step emits drafts[:a] and target[a], the next
  last token is target[a], the length grows by a + 1;
* every row the acceptance reads (0..a) clears the margin;
* the b1_ctx8k draws reach every accept length 0..k and average about the
  recipe's E[a + 1] = (1 - 0.8^5) / 0.2 = 3.36 emitted tokens per step."""
import json
import os

import numpy as np
import pytest

from speculative_decoding_verification_91_b200.inputs import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, f"verify_{name}.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("name", ["b1_ctx8k", "b8_ragged", "b64_6layer"])
def test_fixture_follows_the_recipe_and_the_acceptance_rule(name):
    fx = _load(name)
    wl = W.get_workload(name)
    k, q = wl.k, wl.k + 1
    draws = fx.get("mode") == "draws"
    for s in fx["sequences"]:
        b = s["b"]
        r = W.rejection_point(wl, b, 0 if draws else s["attempt"])
        assert s["r"] == r, (name, b)
        tg = [int(x) for x in s["target_ids"]]
        assert len(tg) == q
        # drafts[< r] are the greedy (= target) tokens, drafts[r] differs
        drafts, r2 = W.make_drafts(wl, b, s["attempt"], np.asarray(tg), r=r)
        assert r2 == r and [int(x) for x in drafts] == [int(x) for x in s["drafts"]], (name, b)
        # the acceptance rule on the stored target ids
        a = next((i for i in range(k) if int(s["drafts"][i]) != tg[i]), k)
        assert s["accept_len"] == a == min(r, k), (name, b)
        emitted = [int(x) for x in s["drafts"][:a]] + [tg[a]]
        assert [int(x) for x in s["emitted"][:a + 1]] == emitted
        assert s["next_last_token"] == tg[a]
        assert s["new_len"] == s["L"] + a + 1
        assert all(s["margin_ok"][: a + 1]), (name, b)
        for i in range(a + 1):
            assert s["top1"][i] - s["top2"][i] >= 0.0


def test_b1_ctx8k_draws_cover_every_accept_length():
    fx = _load("b1_ctx8k")
    assert fx["mode"] == "draws"
    wl = W.get_workload("b1_ctx8k")
    a = [s["accept_len"] for s in fx["sequences"]]
    assert len(a) == 24
    assert set(a) == set(range(wl.k + 1))
    mean = float(np.mean(np.asarray(a) + 1))
    assert mean == pytest.approx(3.25)
    expect = (1 - wl.accept[1] ** (wl.k + 1)) / (1 - wl.accept[1])
    assert abs(mean - expect) < 0.5            # 24 draws of a geometric law capped at k
