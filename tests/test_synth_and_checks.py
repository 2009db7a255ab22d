"""The seeded generator and the parity checkers themselves (no GPU)."""
import numpy as np
import pytest

import synth
from parity_util import check_topk_row, score_error_bound


def test_chunked_generation_is_consistent():
    sp = synth.TensorSpec(7, 3, (1000, 4, 8), 0.5, True)
    full = sp.full()
    np.testing.assert_array_equal(sp.rows(250, 777), full[250:777])
    np.testing.assert_array_equal(sp.take([999, 3, 512]), full[[999, 3, 512]])
    np.testing.assert_array_equal(synth.round_to_bf16(full), full)  # already bf16 values
    assert full.std() == pytest.approx(0.5, rel=0.05)


def test_bf16_rounding_ties_to_even():
    a = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -9, 3.0e-3], dtype=np.float32)
    r = synth.round_to_bf16(a)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] == -1.0
    assert abs(r[4] - 3.0e-3) <= 3.0e-3 * 2 ** -8


def test_workload_inputs_have_the_configured_shapes():
    w = synth.WORKLOADS["tiny_csa_f32"]
    x = synth.make_inputs(w)
    assert x["q"].shape == (1, 512, 8, 128) and x["kv"].shape == (1, 512, 128)
    assert x["qI"].shape == (1, 512, 4, 64) and x["bias"].shape == (8, 128)
    qi, qp = synth.positions(synth.WORKLOADS["csa_decode_bf16"])
    assert qi.shape == (64, 1) and qi.min() >= 131072 - 1024 and qi.max() <= 131071


def test_strided_selection_is_valid():
    w = synth.WORKLOADS["tiny_csa_f32"]
    qi, _ = synth.positions(w)
    idx = synth.strided_selection(w, qi)
    for s in range(w.S):
        vis = min((s + 1) // w.m, w.P_cap)
        n = min(w.topk, vis)
        row = idx[0, s]
        assert np.all(row[n:] == -1) and np.all(np.diff(row[:n]) > 0)
        assert n == 0 or (row[0] >= 0 and row[n - 1] < vis)


def test_topk_checker_catches_wrong_sets():
    rng = np.random.default_rng(0)
    scores = rng.standard_normal(100)
    err = np.zeros(100)
    good = np.sort(np.argsort(-scores, kind="stable")[:10])
    row = np.concatenate([good, -np.ones(2, dtype=int)])
    assert check_topk_row(row[:10], scores, 10, err) == 0
    worst = np.argmin(scores)
    bad = np.sort(np.concatenate([good[1:], [worst]]))
    with pytest.raises(AssertionError):
        check_topk_row(bad, scores, 10, err)
    with pytest.raises(AssertionError):
        check_topk_row(good[::-1], scores, 10, err)         # not ascending
    with pytest.raises(AssertionError):
        check_topk_row(np.concatenate([good[:9], [-1]]), scores, 10, err)
    # a swap across an exact tie is excused only inside the error band
    tied = scores.copy()
    order = np.argsort(-tied, kind="stable")
    tied[order[10]] = tied[order[9]] - 1e-9
    swap = np.sort(np.concatenate([order[:9], [order[10]]]))
    assert check_topk_row(swap, tied, 10, np.full(100, 1e-8)) == 1
    with pytest.raises(AssertionError):
        check_topk_row(swap, tied, 10, np.full(100, 1e-12), rel_tie=0.0)


def test_score_error_bound_scales_with_magnitudes():
    q = np.ones((2, 4))
    k = np.ones((3, 4))
    b = score_error_bound(q, np.array([1.0, -2.0]), k, 0.0)
    assert b.shape == (3,) and np.all(b > 0)
    assert np.allclose(score_error_bound(q, np.array([1.0, -2.0]), 2 * k, 0.0), 2 * b)
