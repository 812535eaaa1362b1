"""Host-side measurement logic of bench.py, on CPU: algorithmic bytes by
hand, the roofline's bound choice and arithmetic, the guard that drops a
recorded ncu traffic figure once its kernel's sources change, the parsing of
sampled clocks and throttle reasons, the expected-tokens law of the sweep and
the loop bench's drafter."""
import json
import os
import types

import numpy as np
import pytest

import bench
from speculative_decoding_verification_91_b200.inputs import workloads as W


def test_algorithmic_bytes_of_the_default_workload_by_hand():
    wl = W.get_workload("b1_ctx8k")                  # L 8192, k 4, Hkv 8, D 256
    kv, lm, _ = bench.algorithmic_bytes(wl, [8192])
    # sliding window 1024, separate K/V: keys 7169 .. 8196 (1028), 2*256*2 bytes per token-head
    local = 1028 * 8 * 1024
    # key-equals-value global layer, p = 0.25: keys 0 .. 8196, (256 + 64)*2 bytes per token-head
    glob = 8197 * 8 * 640
    assert bench.attention_bytes(wl, [8192], 0) == local == 8_421_376
    assert bench.attention_bytes(wl, [8192], 1) == glob == 41_968_640
    assert kv == local + glob
    assert lm == 262_144 * 2560 * 2
    assert 640 / 1024 == 1 - 0.375                      # the K=V layer's saving per token-head


def _fake_root(tmp_path, monkeypatch, peaks):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(peaks))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))


def test_roofline_takes_the_slower_bound(tmp_path, monkeypatch):
    _fake_root(tmp_path, monkeypatch, {"hbm_gbs": 6451.8, "bf16_tflops_sustained": 1405.2})
    peak, kind = bench.measured_peaks()
    assert (peak, kind) == (6451.8, "measured")
    few = types.SimpleNamespace(name="x", d_model=2560, vocab=262_144)
    b = few.vocab * few.d_model * 2 + 5 * few.d_model * 2
    r = bench.lm_roofline(few, {"M": 5}, b, 209.4e-6, peak, kind)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6451.8
    assert r["achieved"] == pytest.approx(b / 209.4e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6451.8)
    assert r["traffic"] is None                          # no capture recorded for this name
    many = types.SimpleNamespace(name="y", d_model=3840, vocab=262_144)
    flops = 2.0 * 256 * 3840 * 262_144                   # 515 GFLOP: 366 us at 1405 TF/s > 312 us of bytes
    r = bench.lm_roofline(many, {"M": 256}, many.vocab * many.d_model * 2, 458e-6, peak, kind)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1405.2
    assert r["achieved"] == pytest.approx(flops / 458e-6 / 1e12)


def test_fallback_peak_without_measurements(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")


def test_recorded_traffic_is_dropped_once_the_kernel_changes(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"sources": ["kernel.cu"], "sources_sha1": bench.kernel_sources_sha1(["kernel.cu"]),
             "dram_bytes_per_launch": 1234}
    tf = tmp_path / "traffic.json"
    tf.write_text(json.dumps({"k/w": entry}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tf))
    assert bench.measured_traffic("k/w") == 1234
    assert bench.measured_traffic("other/w") is None
    src.write_text("// version 2\n")
    assert bench.measured_traffic("k/w") is None


def test_committed_traffic_record_names_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key, e in rec.items():
        assert all(os.path.exists(os.path.join(bench.ROOT, p)) for p in e["sources"]), key
        assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]
        assert e["dram_bytes_per_launch"] >= e["algorithmic_bytes_per_launch"]


def test_clock_summary_reports_median_and_active_reasons():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1965, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # before timing
               "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "0, 1890, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1905, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
               "garbled"]
    c.skip = 1
    s = c.summary()
    assert s["sm_mhz"] == 1905.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    c.lines, c.skip = [], 0
    assert c.summary()["reasons"] == ["unsampled"]


def test_expected_tokens_is_the_mean_of_the_accepted_run_plus_one():
    """E[a + 1] for i.i.d. acceptance alpha, a = leading accepted drafts of k:
    the closed form (1 - alpha^(k+1)) / (1 - alpha), and brute force over all
    2^k accept/reject patterns."""
    import itertools
    for alpha in (0.5, 0.8, 0.9):
        for k in (0, 1, 4, 8):
            closed = (1 - alpha ** (k + 1)) / (1 - alpha)
            brute = 0.0
            for pat in itertools.product((0, 1), repeat=k):
                prob = 1.0
                for ok in pat:
                    prob *= alpha if ok else 1 - alpha
                a = next((i for i, ok in enumerate(pat) if not ok), k)
                brute += prob * (a + 1)
            assert bench.expected_tokens(alpha, k) == pytest.approx(closed, rel=1e-12)
            assert brute == pytest.approx(closed, rel=1e-12)


def test_loop_drafter_keeps_the_greedy_token_where_its_coin_says_so():
    """The loop bench's corrupted-greedy drafter: draft i of step s is the
    greedy stream's token at the sequence's emitted position + i when the
    step's seeded flip i is below the acceptance probability, else the
    step's seeded random id; the same step gives the same drafts."""
    wl = W.get_workload("loop_131k")
    p = wl.accept[1]
    stream = [1000 + 3 * i for i in range(200)]
    drafter = bench.loop_drafter(wl, stream)
    kept = total = 0
    for step, emitted in ((0, 0), (1, 5), (7, 40), (30, 150)):
        flips, ids = W.loop_draft_flips(wl, step)
        d = drafter(step, emitted)
        assert d.dtype == np.int32 and d.shape == (wl.k,)
        assert np.array_equal(d, drafter(step, emitted))
        for i in range(wl.k):
            want = stream[emitted + i] if flips[i] < p else int(ids[i])
            assert int(d[i]) == want
            kept += int(flips[i] < p)
            total += 1
    assert 0.5 < kept / total < 1.0           # p = 0.8 over 32 seeded flips
