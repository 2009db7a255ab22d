"""dsv4_sparse_mqa_attn_scores: the attention that selects each query's index list from its
score row itself ("DeepSeek-V4" doc, Hybrid attention (§2.3), CSA item: the top index_topk
entries per query go straight into core attention) against the two calls it stands for,
dsv4_topk_select then dsv4_sparse_mqa_attn.

  index lists: bit-exact (both sides rank the same fp32 values, written here on the host;
               rows are tie-heavy: small integers, +0 and -0, +-inf, one all-equal row),
               and pinned to the oracle's ranking on every row;
  outputs:     bit-exact (the same kernel over the same lists).
Rows with fewer visible entries than topk (the list is 0..vis-1, then -1) are included.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from oracle import dsv4_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from sparse_long_context_csa_b200 import abi, harness
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    return abi, harness


def _tie_heavy_scores(rng, n_rows, P_cap):
    sc = rng.integers(-6, 7, size=(n_rows, P_cap)).astype(np.float32)
    zeros = rng.random((n_rows, P_cap)) < 0.05
    sc[zeros] = np.where(rng.random(int(zeros.sum())) < 0.5, np.float32(-0.0), np.float32(0.0))
    sc[rng.random((n_rows, P_cap)) < 0.001] = np.inf
    sc[rng.random((n_rows, P_cap)) < 0.001] = -np.inf
    sc[0, :] = 3.0  # all equal: the lowest entries win
    return sc


def _spread_scores(rng, n_rows, P_cap):
    """Distinct-ish fp32 scores of a narrow range (the radix digits must resolve low bits)."""
    return (1.0 + rng.random((n_rows, P_cap)) * 1e-3).astype(np.float32)


@pytest.mark.parametrize("B,S,m,P_cap,topk,kind", [
    (1, 8192, 4, 2048, 512, "ties"),    # the CSA prefill shape
    (2, 2048, 1, 2048, 512, "ties"),    # every row length up to the 2048-entry limit
    (1, 1024, 4, 256, 128, "spread"),   # rows shorter and longer than topk, narrow score range
    (3, 600, 2, 300, 64, "ties"),       # ragged: batch of 3, tail tiles, small topk
])
def test_selection_in_attention_equals_two_calls(lib, B, S, m, P_cap, topk, kind):
    abi, harness = lib
    w = synth.WORKLOADS["csa_prefill_bf16"].replace(B=B, S=S, Sq=S, m=m, P_cap=P_cap, topk=topk)
    specs = synth.tensor_specs(w)
    q = synth.reshape(w, "q", specs["q"].full())
    kv = synth.reshape(w, "kv", specs["kv"].full())
    rng = np.random.default_rng(20261203 + S + topk)
    pool = (rng.standard_normal((B, P_cap, w.D)) / np.sqrt(w.D)).astype(np.float32)
    sink = specs["sink"].full()
    qi, qp = synth.positions(w)
    rows = B * S
    sc = _tie_heavy_scores(rng, rows, P_cap) if kind == "ties" else _spread_scores(rng, rows, P_cap)
    params = harness.params_for(w)
    dt = harness.torch_dtype(w)
    d_q = torch.from_numpy(q).to(dt).cuda()
    d_kv = torch.from_numpy(kv).to(dt).cuda()
    d_pool = torch.from_numpy(pool).to(dt).cuda()
    d_sink = torch.from_numpy(sink).cuda()
    d_pos = torch.from_numpy(qp).cuda()
    d_sc = torch.from_numpy(sc).cuda()

    idx1 = torch.full((B, S, topk), -7, dtype=torch.int32, device="cuda")
    out1 = torch.empty((B, S, w.H, w.dv), dtype=dt, device="cuda")
    abi.dsv4_topk_select(params, d_sc, None, idx1)
    abi.dsv4_sparse_mqa_attn(params, d_q, d_kv, d_pool, idx1, d_sink, d_pos, None, out1)
    idx2 = torch.full((B, S, topk), -7, dtype=torch.int32, device="cuda")
    out2 = torch.empty((B, S, w.H, w.dv), dtype=dt, device="cuda")
    abi.dsv4_sparse_mqa_attn_scores(params, d_q, d_kv, d_pool, d_sc, d_sink, d_pos, None, idx2, out2)
    abi.dsv4_device_check()

    g1, g2 = idx1.cpu().numpy(), idx2.cpu().numpy()
    assert np.array_equal(g1, g2), "index lists differ from dsv4_topk_select"
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16)), "outputs differ from the two calls"
    # pin the lists to the oracle's ranking, row by row
    for r in range(rows):
        b, s = divmod(r, S)
        vis = O.visible_entries(s, m, P_cap)
        ranked, _ = O.topk_select_row(sc[r, :vis], topk)
        want = np.full(topk, -1, dtype=np.int64)
        want[:len(ranked)] = np.sort(np.asarray(ranked, dtype=np.int64))
        assert np.array_equal(g2[b, s].astype(np.int64), want), f"row {(b, s)} (vis={vis}) differs from the oracle"


@pytest.mark.parametrize("B,S,P_cap,topk", [(16, 8192, 2048, 512), (7, 4000, 1000, 256)])
def test_selection_in_attention_decode_shapes(lib, B, S, P_cap, topk):
    """One query per sequence at a spread of cache positions, the window in a ring, and a
    workspace, so each query's keys are split over several CTAs (each split selects the same
    list): lists and outputs bit-exact against dsv4_topk_select + dsv4_sparse_mqa_attn, lists
    against the oracle's ranking."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_decode_bf16"].replace(B=B, S=S, P_cap=P_cap, topk=topk, qindex_spread=min(1024, S // 4))
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    rng = np.random.default_rng(20261204 + B)
    sc = _spread_scores(rng, B, P_cap)
    sc[0] = _tie_heavy_scores(rng, 1, P_cap)[0]
    d_sc = torch.from_numpy(sc).cuda()
    ws = torch.empty(max(abi.dsv4_workspace_bytes(params), 256), dtype=torch.uint8, device="cuda")
    dt = harness.torch_dtype(w)
    idx1 = torch.full((B, 1, topk), -7, dtype=torch.int32, device="cuda")
    out1 = torch.empty((B, 1, w.H, w.dv), dtype=dt, device="cuda")
    abi.dsv4_topk_select(params, d_sc, x["q_index"], idx1)
    abi.dsv4_sparse_mqa_attn(params, x["q"], x["win"], x["pool"], idx1, x["sink"], x["qpos"], x["q_index"], out1, ws)
    idx2 = torch.full((B, 1, topk), -7, dtype=torch.int32, device="cuda")
    out2 = torch.empty((B, 1, w.H, w.dv), dtype=dt, device="cuda")
    abi.dsv4_sparse_mqa_attn_scores(params, x["q"], x["win"], x["pool"], d_sc, x["sink"], x["qpos"], x["q_index"],
                                    idx2, out2, ws)
    abi.dsv4_device_check()
    g1, g2 = idx1.cpu().numpy(), idx2.cpu().numpy()
    assert np.array_equal(g1, g2), "index lists differ from dsv4_topk_select"
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16)), "outputs differ from the two calls"
    for b in range(B):
        vis = O.visible_entries(int(host["q_index"][b, 0]), w.m, P_cap)
        ranked, _ = O.topk_select_row(sc[b, :vis], topk)
        want = np.full(topk, -1, dtype=np.int64)
        want[:len(ranked)] = np.sort(np.asarray(ranked, dtype=np.int64))
        assert np.array_equal(g2[b, 0].astype(np.int64), want), f"sequence {b} (vis={vis}) differs from the oracle"


@pytest.mark.parametrize("name,P_cap,topk", [("tiny_csa_f32", 128, 32), ("csa_prefill_bf16", 4096, 512)])
def test_selection_fallback_equals_two_calls(lib, name, P_cap, topk):
    """Where the attention kernel does not select itself (fp32, or rows longer than 2048
    entries), dsv4_sparse_mqa_attn_scores runs dsv4_topk_select and dsv4_sparse_mqa_attn: the
    same lists and outputs, bit for bit."""
    abi, harness = lib
    w0 = synth.WORKLOADS[name]
    S = 512 if name.startswith("tiny") else 2048
    w = w0.replace(S=S, Sq=S, m=max(1, S // P_cap), P_cap=P_cap, topk=topk)
    specs = synth.tensor_specs(w)
    q = synth.reshape(w, "q", specs["q"].full())
    kv = synth.reshape(w, "kv", specs["kv"].full())
    rng = np.random.default_rng(20261205 + P_cap)
    pool = (rng.standard_normal((w.B, P_cap, w.D)) / np.sqrt(w.D)).astype(np.float32)
    sink = specs["sink"].full()
    _, qp = synth.positions(w)
    sc = _spread_scores(rng, w.B * S, P_cap)
    params = harness.params_for(w)
    dt = harness.torch_dtype(w)
    d = [torch.from_numpy(v).to(dt).cuda() for v in (q, kv, pool)]
    d_sink, d_pos, d_sc = torch.from_numpy(sink).cuda(), torch.from_numpy(qp).cuda(), torch.from_numpy(sc).cuda()
    idx1 = torch.full((w.B, S, topk), -7, dtype=torch.int32, device="cuda")
    idx2 = torch.full((w.B, S, topk), -7, dtype=torch.int32, device="cuda")
    out1 = torch.empty((w.B, S, w.H, w.dv), dtype=dt, device="cuda")
    out2 = torch.empty((w.B, S, w.H, w.dv), dtype=dt, device="cuda")
    abi.dsv4_topk_select(params, d_sc, None, idx1)
    abi.dsv4_sparse_mqa_attn(params, d[0], d[1], d[2], idx1, d_sink, d_pos, None, out1)
    abi.dsv4_sparse_mqa_attn_scores(params, d[0], d[1], d[2], d_sc, d_sink, d_pos, None, idx2, out2)
    abi.dsv4_device_check()
    assert torch.equal(idx1, idx2), "index lists differ"
    assert torch.equal(out1, out2), "outputs differ"
