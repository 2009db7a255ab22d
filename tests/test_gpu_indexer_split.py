"""The Lightning Indexer's two halves as separate entry points (dsv4_indexer_scores,
dsv4_topk_select), against the fp64 oracle.

  scores: every visible entry within the a-priori fp32 accumulation bound of the oracle's
          fp64 score; entries past a row's visible count are left as they were (checked
          bit for bit against a sentinel).
  top-k:  bit-exact.  Both sides rank the SAME fp32 score values (written here, on the
          host), so the decision is taken in the same precision and every tie is decided
          by the lower-index rule; the rows are built to be tie-heavy (small integers, +0
          and -0, +-inf) and to cover the cached (<= 40960 visible) and streamed paths.
  split = fused: scores + top-k through the two calls equals dsv4_indexer_topk.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from oracle import dsv4_oracle as O
from parity_util import sample_rows, score_error_bound

pytestmark = pytest.mark.gpu

SENTINEL = np.float32(-1234.5)


@pytest.fixture(scope="module")
def lib():
    from sparse_long_context_csa_b200 import abi, harness
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    return abi, harness


def _indexer_inputs(w):
    sp = synth.cache_specs(w)
    specs = synth.tensor_specs(w)
    x = {k: synth.reshape(w, k, specs[k].full()) for k in ("qI", "wI")}
    x["poolI"] = sp["poolI"].full().reshape(w.B, w.P_cap, w.cI)
    x["q_index"], _ = synth.positions(w)
    return x


@pytest.mark.parametrize("name", ["tiny_csa_f32", "csa_prefill_bf16", "csa_decode_bf16"])
def test_indexer_scores_kernel(lib, name):
    abi, harness = lib
    w = synth.WORKLOADS[name]
    x = _indexer_inputs(w)
    params = harness.params_for(w)
    d = harness.to_device(w, x)
    scores = torch.full((w.B * w.Sq, w.P_cap), float(SENTINEL), dtype=torch.float32, device="cuda")
    abi.dsv4_indexer_scores(params, d["qI"], d["wI"], d["poolI"], d["q_index"], scores)
    abi.dsv4_device_check()
    g = scores.cpu().numpy()
    rows = [(b, s) for b in range(w.B) for s in (sample_rows(w.Sq, 96, 16) if w.Sq > 1 else [0])]
    for b, s in rows:
        t = int(x["q_index"][b, s])
        vis = O.visible_entries(t, w.m, w.P_cap)
        ref = O.indexer_scores_row(x["qI"][b, s], x["wI"][b, s], x["poolI"][b], vis)
        err = score_error_bound(x["qI"][b, s], x["wI"][b, s], x["poolI"][b][:vis], 0.0)
        row = g[b * w.Sq + s]
        bad = np.abs(row[:vis].astype(np.float64) - ref) > err
        assert not bad.any(), f"{name} row {(b, s)}: {int(bad.sum())} scores outside the fp32 bound"
        assert (row[vis:] == SENTINEL).all(), f"{name} row {(b, s)}: entries past vis={vis} were written"


def _tie_heavy_scores(rng, n_rows, P_cap):
    """Scores drawn from a few small integers (many exact ties), with +-0 and +-inf planted."""
    sc = rng.integers(-6, 7, size=(n_rows, P_cap)).astype(np.float32)
    zeros = rng.random((n_rows, P_cap)) < 0.05
    sc[zeros] = np.where(rng.random(int(zeros.sum())) < 0.5, np.float32(-0.0), np.float32(0.0))
    sc[rng.random((n_rows, P_cap)) < 0.001] = np.inf
    sc[rng.random((n_rows, P_cap)) < 0.001] = -np.inf
    sc[0, :] = 3.0  # one row of all-equal scores: the lowest indices win
    return sc


@pytest.mark.parametrize("P_cap,topk", [(70001, 2048), (9000, 512), (2100, 2048)])
def test_topk_select_bit_exact(lib, P_cap, topk):
    abi, harness = lib
    # m = 1 so that the visible count of cache index t is t + 1: rows below, at and above
    # topk, around the 40960-key shared-memory cache, and the full pool.
    vis_list = sorted({1, topk - 1, topk, topk + 1, min(P_cap, 5000), min(P_cap, 40960),
                       min(P_cap, 40961), P_cap - 1, P_cap})
    vis_list = [P_cap] + vis_list  # row 0: all-equal scores over the whole pool
    B, Sq = 1, len(vis_list)
    q_index = np.array([[v - 1 for v in vis_list]], dtype=np.int32)
    rng = np.random.default_rng(20261202)
    sc = _tie_heavy_scores(rng, Sq, P_cap)
    w = synth.WORKLOADS["csa_decode_bf16"].replace(B=B, Sq=Sq, S=P_cap, m=1, P_cap=P_cap, topk=topk)
    params = harness.params_for(w)
    dsc = torch.from_numpy(sc).cuda()
    dqi = torch.from_numpy(q_index).cuda()
    idx = torch.full((B, Sq, topk), -7, dtype=torch.int32, device="cuda")
    abi.dsv4_topk_select(params, dsc, dqi, idx)
    abi.dsv4_device_check()
    g = idx.cpu().numpy()[0]
    for s in range(Sq):
        t = int(q_index[0, s])
        vis = O.visible_entries(t, 1, P_cap)
        ranked, _ = O.topk_select_row(sc[s, :vis], topk)
        want = np.full(topk, -1, dtype=np.int64)
        want[:len(ranked)] = np.sort(np.asarray(ranked, dtype=np.int64))
        assert np.array_equal(g[s].astype(np.int64), want), f"row {s} (vis={vis}) differs from the oracle"


@pytest.mark.parametrize("topk", [512, 2048])
def test_topk_select_many_long_rows_bit_exact(lib, topk):
    """Hundreds of rows longer than 4096 entries take the path that re-reads each row from its
    scores (256 threads per row, several rows per SM): each warp lists the entries of its
    segment at or above the threshold digit, and the rest of the selection goes over the lists.
    Row kinds: tie-heavy (small integers: lists of tied keys; an all-equal row, whose lists
    overflow and whose threshold digit holds one value); narrow-range distinct scores (every
    key in one digit: the lists overflow and the row is read again digit by digit); the
    one-head indexer's shape, w * ReLU(x) with half of the entries an exact +0 or -0 (w > 0:
    short lists; w < 0: the kept entries are the first exact zeros); decreasing scores, whose
    kept entries all sit in the first warps' segments; and two kinds that defeat a threshold
    taken from a sample of the first 32 entries of every 256 (peaks only where the sample does
    not look: too many entries at or above it; peaks only where it looks: too few), so those
    rows start again on the general path.  Every row against the oracle's ranking."""
    abi, harness = lib
    P_cap, Sq = 9000, 700
    rng = np.random.default_rng(20261203 + topk)
    q_index = rng.integers(0, P_cap, size=(1, Sq)).astype(np.int32)
    q_index[0, :6] = [P_cap - 1, topk - 1, topk, 4096, P_cap - 1, P_cap - 1]
    sc = _tie_heavy_scores(rng, Sq, P_cap)
    kind = rng.integers(0, 6, size=Sq)
    kind[:8] = [0, 1, 0, 0, 2, 3, 4, 5]
    q_index[0, 6:8] = P_cap - 1
    spread = kind == 1
    sc[spread] = (1.0 + rng.random((int(spread.sum()), P_cap)) * 1e-3).astype(np.float32)
    relu = kind == 2
    x = rng.standard_normal((int(relu.sum()), P_cap)).astype(np.float32)
    wsign = np.where(rng.random((int(relu.sum()), 1)) < 0.5, np.float32(-1.5), np.float32(1.5))
    sc[relu] = (wsign * np.maximum(x, np.float32(0.0))).astype(np.float32)  # -1.5 * 0 = -0
    dec = kind == 3
    sc[dec] = (np.float32(1e4) - np.arange(P_cap, dtype=np.float32))[None, :]
    in_sample = (np.arange(P_cap) % 256) < 32
    for k, where in ((4, ~in_sample & (np.arange(P_cap) % 5 == 0)), (5, in_sample)):
        rows = kind == k
        base = (rng.standard_normal((int(rows.sum()), P_cap)) * 0.01).astype(np.float32)
        peak = (10.0 + rng.standard_normal((int(rows.sum()), P_cap))).astype(np.float32)
        sc[rows] = np.where(where[None, :], peak, base)
    w = synth.WORKLOADS["csa_decode_bf16"].replace(B=1, Sq=Sq, S=P_cap, m=1, P_cap=P_cap, topk=topk)
    params = harness.params_for(w)
    idx = torch.full((1, Sq, topk), -7, dtype=torch.int32, device="cuda")
    abi.dsv4_topk_select(params, torch.from_numpy(sc).cuda(), torch.from_numpy(q_index).cuda(), idx)
    abi.dsv4_device_check()
    g = idx.cpu().numpy()[0]
    for s in range(Sq):
        vis = O.visible_entries(int(q_index[0, s]), 1, P_cap)
        ranked, _ = O.topk_select_row(sc[s, :vis], topk)
        want = np.full(topk, -1, dtype=np.int64)
        want[:len(ranked)] = np.sort(np.asarray(ranked, dtype=np.int64))
        assert np.array_equal(g[s].astype(np.int64), want), f"row {s} (vis={vis}) differs from the oracle"


@pytest.mark.parametrize("name", ["tiny_csa_f32", "csa_decode_bf16"])
def test_split_calls_equal_fused_call(lib, name):
    abi, harness = lib
    w = synth.WORKLOADS[name]
    x = _indexer_inputs(w)
    params = harness.params_for(w)
    d = harness.to_device(w, x)
    scores = torch.empty((w.B * w.Sq, w.P_cap), dtype=torch.float32, device="cuda")
    idx_a = torch.empty((w.B, w.Sq, w.topk), dtype=torch.int32, device="cuda")
    idx_b = torch.empty_like(idx_a)
    abi.dsv4_indexer_scores(params, d["qI"], d["wI"], d["poolI"], d["q_index"], scores)
    abi.dsv4_topk_select(params, scores, d["q_index"], idx_a)
    ws = torch.empty(max(abi.dsv4_workspace_bytes(params), 256), dtype=torch.uint8, device="cuda")
    abi.dsv4_indexer_topk(params, d["qI"], d["wI"], d["poolI"], d["q_index"], idx_b, ws)
    abi.dsv4_device_check()
    assert torch.equal(idx_a, idx_b)


@pytest.mark.parametrize("B,S,P_cap,topk,spread", [(64, 131072, 32768, 2048, 1024), (48, 100000, 24576, 2048, 99990),
                                                    (128, 40000, 10000, 512, 39990)])
def test_fused_decode_indexer_matches_the_two_kernel_path(lib, B, S, P_cap, topk, spread):
    """One query per sequence (decode) at a million scored entries or more: dsv4_indexer_topk
    scores and selects in one kernel (split top-k in each CTA, merged by the last CTA of each
    query).  Its index lists must equal, bit for bit, those of the two separate kernels
    (dsv4_indexer_scores, then dsv4_topk_select) on the same inputs.  Three queries are moved
    to the start of their caches (no visible entry, or one); the wider spreads put more below
    topk visible entries."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_decode_bf16"].replace(B=B, S=S, P_cap=P_cap, topk=topk, qindex_spread=spread)
    sp = synth.cache_specs(w)
    specs = synth.tensor_specs(w)
    qi, _ = synth.positions(w)
    qi[:3, 0] = [0, 2, 3]  # two queries with no visible entry yet, one with a single entry
    host = {"qI": synth.reshape(w, "qI", specs["qI"].full()), "wI": synth.reshape(w, "wI", specs["wI"].full()),
            "poolI": sp["poolI"].full().reshape(w.B, w.P_cap, w.cI), "q_index": qi}
    p = harness.params_for(w)
    d = harness.to_device(w, host)
    ws = torch.empty(max(abi.dsv4_workspace_bytes(p), 256), dtype=torch.uint8, device="cuda")
    fused = torch.full((w.B, 1, w.topk), -7, dtype=torch.int32, device="cuda")
    for _ in range(2):  # twice: the per-query split counters must be left ready for the next call
        abi.dsv4_indexer_topk(p, d["qI"], d["wI"], d["poolI"], d["q_index"], fused, ws)
    scores = torch.empty((w.B, w.P_cap), dtype=torch.float32, device="cuda")
    split = torch.full((w.B, 1, w.topk), -7, dtype=torch.int32, device="cuda")
    abi.dsv4_indexer_scores(p, d["qI"], d["wI"], d["poolI"], d["q_index"], scores)
    abi.dsv4_topk_select(p, scores, d["q_index"], split)
    abi.dsv4_device_check()
    assert torch.equal(fused, split)
    vis = np.minimum((qi[:, 0] + 1) // w.m, w.P_cap)
    kept = (fused.cpu().numpy()[:, 0] >= 0).sum(axis=1)
    np.testing.assert_array_equal(kept, np.minimum(vis, w.topk))
