"""Comparison helpers for the GPU-vs-oracle parity tests (no arithmetic of the method)."""
from __future__ import annotations

import numpy as np

U32 = 2.0 ** -24  # unit roundoff of fp32


def sample_rows(n: int, k: int = 512, edge: int = 64) -> list[int]:
    """Strided sample of k row ids plus the first and last `edge` rows."""
    rows = set(range(min(edge, n))) | set(range(max(0, n - edge), n))
    if n > 0:
        rows |= set(np.linspace(0, n - 1, min(k, n)).astype(int).tolist())
    return sorted(rows)


def score_error_bound(qI_t, wI_t, keys, rel_key_err: float) -> np.ndarray:
    """A-priori bound on |fp32 score - exact score| per entry.

    The kernel accumulates cI bf16/fp32 products in fp32 per head and sums nI weighted
    heads: |err| <= (cI + nI + 2) u * sum_h |w_h| sum_d |q_hd k_d|.  ``rel_key_err``
    adds the effect of key values that may differ from the oracle's by that relative
    amount (storage rounding of a pool both sides computed).
    """
    qI_t = np.asarray(qI_t, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    mag = np.abs(keys) @ np.abs(qI_t).T              # [vis, nI]
    mag = mag @ np.abs(np.asarray(wI_t, dtype=np.float64))  # [vis]
    cI, nI = qI_t.shape[1], qI_t.shape[0]
    return mag * ((cI + nI + 2) * U32 + rel_key_err)


def check_topk_row(gpu_row, scores, K, err, rel_tie=1e-6, stats=None):
    """Check a GPU top-k row against fp64 scores of the visible entries.

    Rules: the row holds min(K, vis) distinct visible entries in ascending order, then -1;
    it equals the oracle's set except for entries whose score is within the combined
    error band of the K-th score (near ties the two precisions may break differently).
    Returns the number of excused differences; raises AssertionError otherwise.

    ``stats`` (a dict, optional) accumulates: rows checked, rows with a swap, swapped
    entries, and swapped entries whose fp64 gap to the K-th score exceeds ``rel_tie``
    relative (excused only by the fp32 accumulation band, not by the 1e-6 rule).
    """
    gpu_row = np.asarray(gpu_row)
    vis = scores.shape[0]
    n = min(K, vis)
    sel = gpu_row[:n]
    if stats is not None:
        stats["rows"] = stats.get("rows", 0) + 1
    assert np.all(gpu_row[n:] == -1), "slots past min(K, vis) must be -1"
    assert np.all((sel >= 0) & (sel < vis)), "selected entry not visible"
    assert np.all(np.diff(sel) > 0), "entries must be distinct and ascending"
    if vis <= K:
        assert np.array_equal(sel, np.arange(vis)), "with vis <= K every entry is kept"
        return 0
    order = np.lexsort((np.arange(vis), -scores))
    ref = np.sort(order[:K])
    if np.array_equal(ref, sel):
        return 0
    kth = scores[order[K - 1]]
    band = np.maximum(err, rel_tie * abs(kth))
    extra = np.setdiff1d(sel, ref)
    missing = np.setdiff1d(ref, sel)
    beyond = 0
    for w_ in np.concatenate([extra, missing]):
        gap = abs(scores[w_] - kth)
        assert gap <= band[w_] + band[order[K - 1]], (
            f"entry {w_} differs (score {scores[w_]!r}, K-th {kth!r}, band {band[w_]!r})")
        beyond += int(gap > rel_tie * abs(kth))
    if stats is not None:
        stats["rows_with_swaps"] = stats.get("rows_with_swaps", 0) + 1
        stats["swapped_entries"] = stats.get("swapped_entries", 0) + len(extra) + len(missing)
        stats["swaps_beyond_1e-6_rel"] = stats.get("swaps_beyond_1e-6_rel", 0) + beyond
    return len(extra)


def report(name, stats):
    """One line of near-tie statistics (shown with pytest -s)."""
    print(f"[near-ties] {name}: {stats.get('rows', 0)} rows, {stats.get('rows_with_swaps', 0)} with a swap, "
          f"{stats.get('swapped_entries', 0)} swapped entries, "
          f"{stats.get('swaps_beyond_1e-6_rel', 0)} of them beyond 1e-6 relative")


def assert_close_rel(got, ref, rtol, atol=0.0, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    lim = rtol * np.abs(ref) + atol
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (rtol {rtol}, atol {atol})")


def assert_max_abs(got, ref, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    m = float(err.max()) if err.size else 0.0
    assert m <= tol, f"{what}: max abs error {m:.3e} > {tol:.1e} at {np.unravel_index(np.argmax(err), err.shape)}"
    return m
