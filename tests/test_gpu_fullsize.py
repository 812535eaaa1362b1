"""Full-size verify steps against oracle fixtures (tests/golden/verify_*.json,
written by tests/golden/make_golden.py from the oracle alone), in the same
launch configuration the benchmark times (spec_verify_step on one session)."""
import glob
import json
import os

import numpy as np
import pytest
import torch

from speculative_decoding_verification_91_b200 import binding as B
from speculative_decoding_verification_91_b200.inputs import workloads as W
from speculative_decoding_verification_91_b200.session import WorkloadSession

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FIXTURES = sorted(os.path.basename(p)[len("verify_"):-len(".json")]
                  for p in glob.glob(os.path.join(GOLDEN, "verify_*.json")))
ATOL, RTOL = 2e-2, 1e-2


@pytest.mark.parametrize("name", FIXTURES)
def test_full_size_step_matches_oracle(name):
    """Fixtures in draws mode hold independent batch-1 steps (draw b seeded as
    sequence b); each runs alone, as the benchmark times it.  Other fixtures
    run as one batched step."""
    with open(os.path.join(GOLDEN, f"verify_{name}.json")) as f:
        fx = json.load(f)
    seqs = fx["sequences"]
    draws = fx.get("mode") == "draws"
    wl = W.get_workload(fx["workload"])
    if draws:
        wl = wl.with_(batch=len(seqs))
    s = WorkloadSession(wl, attempts=[q["attempt"] for q in seqs])
    s.set_inputs([q["last_token"] for q in seqs],
                 np.array([q["drafts"] for q in seqs], dtype=np.int32) if wl.k else [])
    for rep in range(2):        # a second identical step: counters and status were left clean
        s.reset_lengths()
        if draws:
            for b in range(len(seqs)):
                s.step_one(b)
        else:
            s.step()
        out = s.outputs()
        assert s.ws.device_status() == 0
        for b, q in enumerate(seqs):
            a = q["accept_len"]
            assert out["accept_len"][b] == a
            assert out["emitted"][b].tolist() == q["emitted"]
            assert out["new_last"][b] == q["next_last_token"]
            assert out["seq_lens"][b] == q["new_len"]
            for i in range(wl.q_rows):
                t1 = q["top1"][i]
                assert abs(out["target_max"][b][i] - t1) <= ATOL + RTOL * abs(t1), (b, i)
                if q["margin_ok"][i]:
                    assert out["target_ids"][b][i] == q["target_ids"][i], (b, i)
    if draws:                   # the draws exercise acceptance at full size
        assert max(q["accept_len"] for q in seqs) >= 1
