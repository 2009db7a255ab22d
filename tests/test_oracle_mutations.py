"""The oracle's pins catch plausible mistakes: each case below plants one mistake in a copy of
the oracle's source (text replacement, compiled into a throw-away module on the CPU; the real
module is untouched) and checks that at least one named pin from test_oracle_pins fails on it.

A replacement must match the oracle source exactly once, so that a change of the oracle that
moves the planted site fails here loudly instead of silently testing nothing.
"""
from __future__ import annotations

import os
import types

import pytest

import test_oracle_pins as pins

SRC_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "dsv4_oracle.py")
SRC = open(SRC_PATH).read()

# (name, text in the oracle, planted replacement, pins expected to catch it: (test, kwargs))
MUTATIONS = [
    ("sink dropped from the denominator",
     "denom = e.sum(axis=1) + np.exp(sink - mx)", "denom = e.sum(axis=1)",
     [("test_sink_is_an_extra_logit_with_zero_value", {}), ("test_single_key_closed_form", {})]),
    ("rotation sign",
     "out[..., c - R::2] = a * cos - b * sin", "out[..., c - R::2] = a * cos + b * sin",
     [("test_rope_closed_form_and_algebra", {})]),
    ("rope pair order",
     "a = x[..., c - R::2]\n    b = x[..., c - R + 1::2]", "a = x[..., c - R + 1::2]\n    b = x[..., c - R::2]",
     [("test_rope_closed_form_and_algebra", {})]),
    ("rope frequency exponent",
     "inv_freq = float(theta) ** (-2.0 * k / R)", "inv_freq = float(theta) ** (-1.0 * k / R)",
     [("test_rope_closed_form_and_algebra", {})]),
    ("sliding window one token too long",
     "return list(range(max(0, t - n_win + 1), t + 1))", "return list(range(max(0, t - n_win), t + 1))",
     [("test_mask_example_grid", {})]),
    ("entry visible one token early",
     "v = (t + 1) // m", "v = (t + 2) // m",
     [("test_mask_example_grid", {})]),
    ("tie rule: higher index wins",
     "order = np.lexsort((np.arange(vis), -scores))", "order = np.lexsort((-np.arange(vis), -scores))",
     [("test_topk_brute_force_with_ties", {"seed": s}) for s in range(6)]),
    ("overlap window geometry",
     "lo = (w - 1) * m if overlap else w * m\n    hi = (w + 1) * m",
     "lo = (w - 2) * m if overlap else w * m\n    hi = (w + 1) * m",
     [("test_compress_zero_logits_is_window_mean", {"overlap": 1}),
      ("test_compress_gate_selects_and_slot_bias_alignment", {"overlap": 1})]),
    ("entry rotated at the last token of its block",
     "entry = rope_rotate(entry, pos[b, w * m], R, theta)", "entry = rope_rotate(entry, pos[b, w * m + m - 1], R, theta)",
     [("test_compress_rope_position_is_first_token_of_own_block", {})]),
    ("softmax scale not applied",
     "logits = scale * (q_rot @ keys.T)", "logits = (q_rot @ keys.T)",
     [("test_single_key_closed_form", {}), ("test_hca_equals_dense_masked_attention", {})]),
    ("indexer without the ReLU",
     "return (np.maximum(dots, 0.0) * wI_t[None, :]).sum(axis=1)", "return (dots * wI_t[None, :]).sum(axis=1)",
     [("test_indexer_hand_example", {})]),
    ("compressor softmax over channels instead of tokens",
     "            alpha = e / e.sum(axis=0)\n            entry = (alpha * x[b, js]).sum(axis=0)",
     "            alpha = e / e.sum(axis=1, keepdims=True)\n            entry = (alpha * x[b, js]).sum(axis=0)",
     [("test_compress_zero_logits_is_window_mean", {"overlap": 1}),
      ("test_compress_gate_selects_and_slot_bias_alignment", {"overlap": 1}),
      ("test_compress_is_linear_in_the_rows_and_its_weights_sum_to_one", {})]),
    ("per-slot bias in reversed slot order",
     "logit = logit + bias[slots]", "logit = logit + bias[slots[::-1]]",
     [("test_compress_gate_selects_and_slot_bias_alignment", {"overlap": 1}),
      ("test_compress_gate_selects_and_slot_bias_alignment", {"overlap": 0})]),
    ("sliding layer keys rotated one position late",
     "kv_rot = store_as(rope_rotate(kv, pos, R, theta), store)\n    q_index = np.tile(np.arange(S), (B, 1))\n    out = sparse_mqa_attention(q, kv_rot, np.zeros((B, 0, D))",
     "kv_rot = store_as(rope_rotate(kv, pos + 1, R, theta), store)\n    q_index = np.tile(np.arange(S), (B, 1))\n    out = sparse_mqa_attention(q, kv_rot, np.zeros((B, 0, D))",
     [("test_sliding_layer_equals_dense_window_attention", {}), ("test_sliding_layer_follows_the_worked_mask", {})]),
    ("output-projection groups interleaved instead of contiguous heads",
     "o[:, i * hg:(i + 1) * hg, :].reshape(T, hg * dv)", "o[:, i::g, :].reshape(T, hg * dv)",
     [("test_grouped_out_proj_equals_dense_block_diagonal_product", {}), ("test_grouped_out_proj_special_cases", {})]),
    ("decode cache buffer slot off by one",
     'cache["raw"][t % lw] = _f64(x_t)', 'cache["raw"][(t + 1) % lw] = _f64(x_t)',
     [("test_decode_append_matches_prefill_compression", {"m": 4, "overlap": True})]),
    ("decode cache entry rotated at the newest token",
     'entry = rope_rotate(entry, cache["pos"][(w * m) % lw], R, theta)',
     'entry = rope_rotate(entry, cache["pos"][t % lw], R, theta)',
     [("test_decode_append_matches_prefill_compression", {"m": 4, "overlap": True})]),
    ("bf16 storage truncates instead of rounding",
     "r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16", "r = (u >> 16).astype(np.uint32) << 16",
     [("test_store_as_bf16_rounds_to_nearest_even", {}), ("test_store_as_matches_library_conversions", {})]),
    ("bf16 storage rounds ties away from zero (tie-to-even term dropped)",
     "u + 0x7FFF + ((u >> 16) & 1)", "u + 0x8000",
     [("test_store_as_bf16_rounds_to_nearest_even", {}), ("test_store_as_matches_library_conversions", {})]),
]


def _mutant(old: str, new: str) -> types.ModuleType:
    assert SRC.count(old) == 1, f"planted site not found exactly once: {old!r}"
    mod = types.ModuleType("dsv4_oracle_mutant")
    exec(compile(SRC.replace(old, new), "dsv4_oracle_mutant", "exec"), mod.__dict__)
    return mod


def test_unmutated_copy_passes_the_pins(monkeypatch):
    """Control: the compiled copy of the unchanged source passes every pin used below."""
    mod = types.ModuleType("dsv4_oracle_copy")
    exec(compile(SRC, "dsv4_oracle_copy", "exec"), mod.__dict__)
    monkeypatch.setattr(pins, "O", mod)
    for _, _, _, checks in MUTATIONS:
        for name, kwargs in checks:
            getattr(pins, name)(**kwargs)


@pytest.mark.parametrize("name,old,new,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, old, new, checks):
    monkeypatch.setattr(pins, "O", _mutant(old, new))
    failed = []
    for test_name, kwargs in checks:
        try:
            getattr(pins, test_name)(**kwargs)
        except (AssertionError, ValueError, IndexError):
            failed.append(test_name)
    assert failed, f"planted mistake '{name}' passed every pin {[c[0] for c in checks]}"
