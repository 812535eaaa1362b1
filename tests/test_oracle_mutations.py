"""Planted mistakes in the oracle (CPU only).

Each case changes one expression of one oracle function — a sign, an index,
an axis, a comparison, a dropped term, swapped operands — the kind of slip a
restatement of the pages could contain, and checks that at least one of the
pins named for it fails.  The mistake is planted in a patched copy of the
oracle function for the duration of the case; the oracle's files are not
touched.  A control case runs the same pins unplanted and requires them all
to pass, so a detection is never a pin that fails anyway.
"""
import __future__
import inspect
import textwrap

import pytest

import oracle
from oracle import draft as OD
from oracle import sampled as OS
from oracle import verify as OV

from . import test_oracle as T
from . import test_oracle_draft as TD
from . import test_oracle_sampled as TS

_MODULES = (oracle, OV, OD, OS)


def _plant(monkeypatch, module, name, old, new):
    """Replace `old` by `new` (exactly one occurrence) in the source of
    module.name and install the result wherever the oracle binds that name."""
    fn = getattr(module, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, f"{name}: {old!r} must occur exactly once"
    ns = dict(vars(module))
    code = compile(src.replace(old, new), f"<planted {name}>", "exec",
                   flags=__future__.annotations.compiler_flag, dont_inherit=True)
    exec(code, ns)
    planted = ns[name]
    for m in _MODULES:
        if getattr(m, name, None) is fn:
            monkeypatch.setattr(m, name, planted)


def _pin(f, *args):
    return (f, args)


# (case, module, function, old, new, pins that should catch it)
CASES = [
    # ---- RoPE / p-RoPE
    ("rope_sign", OV, "rope", "x[..., :n] = (a * c) - (b * s)", "x[..., :n] = (a * c) + (b * s)",
     [_pin(T.test_rope_equals_complex_rotation, 256, 0.25), _pin(T.test_rope_relative_position_and_norm)]),
    ("rope_pair_partner", OV, "rope", "b = x[..., h:h + n].copy()", "b = x[..., h - 1:h - 1 + n].copy()",
     [_pin(T.test_rope_equals_complex_rotation, 128, 1.0)]),
    ("rope_frequency_exponent", OV, "rope_inv_freq", "-2.0 * i / head_dim", "-1.0 * i / head_dim",
     [_pin(T.test_rope_equals_complex_rotation, 128, 1.0), _pin(T.test_p_rope_rotates_only_highest_frequency_quarter)]),
    ("p_rope_lowest_frequencies", OV, "rope_cos_sin", "[None, :n]", "[None, -n:]",
     [_pin(T.test_rope_equals_complex_rotation, 256, 0.25)]),
    ("p_rope_pair_count", OV, "rope_rotated_pairs", "fraction * head_dim / 2", "fraction * head_dim",
     [_pin(T.test_p_rope_rotates_only_highest_frequency_quarter),
      _pin(T.test_key_equals_value_cache_saving_is_37_5_percent)]),
    # ---- RMSNorm
    ("rmsnorm_eps_dropped", OV, "rmsnorm", "keepdims=True) + eps)", "keepdims=True))",
     [_pin(T.test_rmsnorm_closed_forms)]),
    ("rmsnorm_axis", OV, "rmsnorm", "np.mean(x * x, axis=-1", "np.mean(x * x, axis=0",
     [_pin(T.test_rmsnorm_closed_forms), _pin(T.test_rmsnorm_matches_torch_layer)]),
    # ---- attention
    ("attend_scale_dropped", OV, "attend", "s = (q @ keys.T) * scale", "s = (q @ keys.T)",
     [_pin(T.test_attend_matches_torch_sdpa, 0), _pin(T.test_attend_special_cases)]),
    ("attend_window_off_by_one", OV, "attend", "vis &= kpos[None, :] > qpos[:, None] - window",
     "vis &= kpos[None, :] >= qpos[:, None] - window",
     [_pin(T.test_attend_matches_torch_sdpa, 5), _pin(T.test_attend_special_cases)]),
    ("attend_causal_excludes_self", OV, "attend", "vis = kpos[None, :] <= qpos[:, None]",
     "vis = kpos[None, :] < qpos[:, None]",
     [_pin(T.test_attend_matches_torch_sdpa, 0), _pin(T.test_attend_special_cases)]),
    ("attend_max_axis", OV, "attend", "m = s.max(axis=1, keepdims=True)", "m = s.max(axis=0, keepdims=True)",
     [_pin(T.test_attend_matches_torch_sdpa, 0)]),
    ("attend_not_normalised", OV, "attend", "return (p @ vals) / p.sum(axis=1, keepdims=True)",
     "return (p @ vals)", [_pin(T.test_attend_matches_torch_sdpa, 0)]),
    ("gqa_head_mapping", OV, "attention_layer", "kh = h // G", "kh = h % Hkv",
     [_pin(T.test_attention_layer_is_gqa_sdpa, False, 0, 1.0)]),
    ("attention_scale", OV, "attention_layer", "scale = 1.0 / np.sqrt(D)", "scale = 1.0 / D",
     [_pin(T.test_attention_layer_is_gqa_sdpa, False, 0, 1.0)]),
    ("rows_at_wrong_positions", OV, "attention_layer", "pos = np.arange(L, L + nq)",
     "pos = np.arange(L + 1, L + nq + 1)", [_pin(T.test_attention_layer_is_gqa_sdpa, False, 7, 1.0)]),
    # ---- key-equals-value
    ("kv_equal_values_post_rope", OV, "attention_layer", "vals_new = kpre_new", "vals_new = k_new",
     [_pin(T.test_attention_layer_is_gqa_sdpa, True, 0, 0.25)]),
    ("kv_equal_cache_values_post_rope", OV, "cache_from_raw", "return LayerCache(lo, k, None, bf16(k_raw))",
     "return LayerCache(lo, k, None, k)",
     [_pin(T.test_key_equals_value_values_are_recoverable),
      _pin(T.test_attention_layer_is_gqa_sdpa, True, 0, 0.25)]),
    # ---- forward
    ("residual_dropped", OV, "verify_forward", "x = f32(x.astype(np.float64) + y.astype(np.float64))",
     "x = f32(y.astype(np.float64))", [_pin(T.test_forward_degenerate_zero_output_projection)]),
    ("final_norm_dropped", OV, "verify_forward", "h = bf16(rmsnorm(x[rows], model.rms_eps))",
     "h = bf16(x[rows])", [_pin(T.test_forward_degenerate_zero_output_projection)]),
    ("embedding_rows_reversed", OV, "verify_forward", "emb[tokens]", "emb[tokens[::-1]]",
     [_pin(T.test_forward_degenerate_zero_output_projection)]),
    # ---- LM head + argmax
    ("argmax_ties_to_later_chunk", OV, "lm_head_top2", "better = c1 > top1", "better = c1 >= top1",
     [_pin(T.test_lm_head_ties_go_to_lowest_id)]),
    ("runner_up_drops_old_best", OV, "lm_head_top2",
     "new_top2 = np.where(better, np.maximum(top1, c2), np.maximum(top2, c1))",
     "new_top2 = np.where(better, c2, np.maximum(top2, c1))", [_pin(T.test_lm_head_matches_torch_argmax)]),
    # ---- acceptance, commit, loop
    ("accept_compares_next_row", OV, "accept_longest_prefix", "while a < k and drafts[a] == g[a]:",
     "while a < k and drafts[a] == g[a + 1]:",
     [_pin(T.test_accept_cases_from_pages), _pin(T.test_accept_brute_force_over_match_patterns, 3)]),
    ("bonus_from_wrong_row", OV, "accept_longest_prefix", "emitted = drafts[:a] + [g[a]] + [-1] * (k - a)",
     "emitted = drafts[:a] + [g[min(a + 1, k)]] + [-1] * (k - a)",
     [_pin(T.test_accept_cases_from_pages), _pin(T.test_accept_brute_force_over_match_patterns, 3)]),
    ("commit_keeps_the_last_rows", OV, "commit", "np.concatenate([c.k, k[:n_rows]], axis=0)",
     "np.concatenate([c.k, k[k.shape[0] - n_rows:]], axis=0)",
     [_pin(T.test_speculative_loop_equals_greedy_decoding, 0)]),
    ("no_rollback_of_rejected_rows", OV, "speculative_decode",
     "caches = commit(caches, res.forward, res.accept_len + 1)", "caches = commit(caches, res.forward, k + 1)",
     [_pin(T.test_speculative_loop_equals_greedy_decoding, 0)]),
    # ---- drafter
    ("draft_query_position", OD, "draft_step", "L, L + s, q_pre)", "L, L + s + 1, q_pre)",
     [_pin(TD.test_draft_step_queries_sit_at_L_plus_s)]),
    # (the window test inside cross_attention is repeated by attend, so
    #  changing only the former is an equivalent mutant; its head mapping is
    #  planted instead)
    ("draft_gqa_head_mapping", OD, "cross_attention", "kh = h // G", "kh = h % Hkv",
     [_pin(TD.test_query_position_is_committed_length_plus_step),
      _pin(TD.test_cross_attention_is_masked_sdpa, 7, False, 1.0, 3)]),
    ("draft_concat_order", OD, "draft_step", "u = np.concatenate([bf16(prev_hidden).astype(np.float64), tok])",
     "u = np.concatenate([tok, bf16(prev_hidden).astype(np.float64)])",
     [_pin(TD.test_projections_and_unembed_when_blocks_add_nothing)]),
    ("cluster_ties_to_higher_id", OD, "cheap_unembed", "key=lambda c: (-cl[c], c)", "key=lambda c: (-cl[c], -c)",
     [_pin(TD.test_cheap_unembed_keeps_the_best_clusters, 3),
      _pin(TD.test_cheap_unembed_tie_at_the_kept_boundary_keeps_the_lower_cluster_id)]),
    ("clusters_kept_are_the_worst", OD, "cheap_unembed", "sel = order[:tables.n_select]",
     "sel = order[len(order) - tables.n_select:]",
     [_pin(TD.test_cheap_unembed_keeps_the_best_clusters, 3)]),
    # ---- sampled verification
    ("accept_ratio_inverted", OS, "speculative_sample", "if u[a] * qd < pd:", "if u[a] * pd < qd:",
     [_pin(TS.test_impossible_draft_is_rejected_and_redrawn_elsewhere)]),
    ("residual_not_subtracted", OS, "speculative_sample", "w = np.maximum(p[a] - qa, 0.0)", "w = p[a]",
     [_pin(TS.test_emitted_tokens_follow_the_target_distribution, 1.0)]),
    ("gumbel_sign", OS, "gumbel_draw", "np.log(w) - np.log(-np.log(g))", "np.log(w) + np.log(-np.log(g))",
     [_pin(TS.test_gumbel_draw_frequencies_follow_the_weights)]),
    ("logits_chunk_misaligned", OS, "full_logits", "out[:, v0:v0 + chunk] = f32(h @ bf16_from_bits(w_bits[v0:v0 + chunk])",
     "out[:, v0:v0 + chunk] = f32(h @ bf16_from_bits(w_bits[v0 + 1:v0 + chunk + 1])",
     [_pin(TS.test_full_logits_match_torch_and_the_argmax_head)]),
    ("temperature_ignored", OS, "softmax", "z = np.asarray(logits, dtype=np.float64) / T",
     "z = np.asarray(logits, dtype=np.float64)", [_pin(TS.test_softmax_temperature_closed_forms)]),
]


def _fails(f, args):
    try:
        f(*args)
    except (AssertionError, ValueError):
        return True
    return False


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_is_caught(case, monkeypatch):
    _, module, name, old, new, pins = case
    _plant(monkeypatch, module, name, old, new)
    caught = [f.__name__ for f, args in pins if _fails(f, args)]
    assert caught, f"no pin caught the planted mistake in {name}: {old!r} -> {new!r}"


def test_pins_pass_without_a_planted_mistake():
    seen = set()
    for _, _, _, _, _, pins in CASES:
        for f, args in pins:
            if (f, args) in seen:
                continue
            seen.add((f, args))
            f(*args)
