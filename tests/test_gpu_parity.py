"""GPU-vs-oracle parity of every step of the hot path, through the C ABI.

Inputs come from ``synth`` (seeded, identical on both sides); expected values come only
from the fp64 oracle.  Tolerances (written here, from the method's targets):
  attention output, max abs error: 1e-5 (fp32 workloads), 2e-3 (bf16 workloads);
  stored pools / rotated rows: within one storage ulp (2^-23 fp32, 2^-7 bf16, relative);
  top-k index sets: bit-exact except entries whose fp64 score lies inside the combined
  error band of the K-th score (near ties), band = max(1e-6 relative, a-priori bound of
  the kernel's fp32 accumulation plus storage-rounding differences of the key pool).
Layer tests compare every sampled attention row: with the oracle's output where the index
sets match, and with the oracle's attention driven by the GPU's index set where they differ
at an excused near tie.  The kernel-level attention tests feed both sides the same seeded
index lists.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from oracle import dsv4_oracle as O
from parity_util import (assert_close_rel, assert_max_abs, check_topk_row, report, sample_rows,
                         score_error_bound)

pytestmark = pytest.mark.gpu

ATTN_TOL = {"f32": 1e-5, "bf16": 2e-3}
STORE_RTOL = {"f32": 2.0 ** -23, "bf16": 2.0 ** -7}
STORE = {"f32": "f32", "bf16": "bf16"}
U32 = 2.0 ** -24


def fp32_atol(x, n_terms):
    """Absolute error bound of an fp32 sum of n_terms products of inputs |x| (weights <= 1),
    which the relative storage tolerance does not cover when the result cancels to ~0."""
    return (n_terms + 8) * U32 * float(np.abs(np.asarray(x)).max())


@pytest.fixture(scope="module")
def lib():
    from sparse_long_context_csa_b200 import abi, harness
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    return abi, harness


def _np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def _run_layer(lib, w, gains=None):
    abi, harness = lib
    host = synth.make_inputs(w, gains)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o = harness.make_outputs(w, params)
    harness.step(w, params, x, o)
    abi.dsv4_device_check()
    return host, o


def _oracle_kw(w):
    return dict(m=w.m, n_win=w.n_win, scale=w.scale, dv=w.dv, R=w.R, theta=w.theta,
                rotate_out=w.rotate_out)


def _check_layer_idx_and_out(w, host, o, ref, rows, rel_key_err, name=None):
    """Top-k rows against oracle scores, then every sampled row's attention output.

    A row whose GPU index set equals the oracle's is compared with the oracle's output; a
    row whose set differs only at excused near ties is compared with the oracle's attention
    driven by the GPU's index set (over the oracle's own stored pool and rotated rows), so
    that a near tie does not cascade into the attention check and no sampled row is skipped.
    """
    gidx = _np(o["idx"])
    gout = _np(o["out"])
    poolI = ref["poolI"]
    q_index = np.tile(np.arange(w.S), (w.B, 1))
    stats, worst = {}, 0.0
    for (b, s) in rows:
        t = s
        vis = O.visible_entries(t, w.m, w.P_cap)
        sc = O.indexer_scores_row(host["qI"][b, s], host["wI"][b, s], poolI[b], vis)
        err = score_error_bound(host["qI"][b, s], host["wI"][b, s], poolI[b][:vis], rel_key_err)
        n = check_topk_row(gidx[b, s], sc, w.topk, err, stats=stats)
        if n == 0:
            want = ref["out"][b, s]
        else:
            want = O.sparse_mqa_attention(host["q"], ref["kv_rot"], ref["pool"], gidx.astype(np.int64),
                                          host["sink"], host["pos"], q_index, rope_q=True, rows=[(b, s)],
                                          **_oracle_kw(w))[b, s]
        worst = max(worst, assert_max_abs(gout[b, s], want, ATTN_TOL[w.dtype], f"out row {(b, s)}"))
    report(name or w.name, stats)
    return stats.get("swapped_entries", 0), worst


# ------------------------------------------------------------------ full layers
@pytest.mark.parametrize("gains", [None, {"q": 64.0, "qI": 8.0}], ids=["plain", "peaky"])
def test_tiny_csa_layer_f32(lib, gains):
    w = synth.WORKLOADS["tiny_csa_f32"]
    host, o = _run_layer(lib, w, gains)
    ref = O.csa_layer(host["q"], host["kv"], host["z"], host["bias"], host["qI"], host["wI"], host["kI"],
                      host["zI"], host["biasI"], host["sink"], host["pos"], overlap=w.overlap, topk=w.topk,
                      store="f32", **_oracle_kw(w))
    P = w.S // w.m
    nt = 2 * w.m if w.overlap else w.m
    assert_close_rel(_np(o["pool"])[:, :P], ref["pool"], STORE_RTOL["f32"], fp32_atol(host["kv"], nt), "pool")
    assert_close_rel(_np(o["poolI"])[:, :P], ref["poolI"], STORE_RTOL["f32"], fp32_atol(host["kI"], nt), "poolI")
    assert_close_rel(_np(o["kv_rot"]), ref["kv_rot"], STORE_RTOL["f32"], fp32_atol(host["kv"], 2), "kv_rot")
    rows = [(0, s) for s in range(w.S)]
    _check_layer_idx_and_out(w, host, o, ref, rows, rel_key_err=4 * 2.0 ** -24)


def test_csa_prefill_layer_bf16(lib):
    w = synth.WORKLOADS["csa_prefill_bf16"]
    host, o = _run_layer(lib, w)
    rows = [(0, s) for s in sample_rows(w.S, 384, 64)]
    ref = O.csa_layer(host["q"], host["kv"], host["z"], host["bias"], host["qI"], host["wI"], host["kI"],
                      host["zI"], host["biasI"], host["sink"], host["pos"], overlap=w.overlap, topk=w.topk,
                      store="bf16", rows=rows, **_oracle_kw(w))
    P = w.S // w.m
    nt = 2 * w.m if w.overlap else w.m
    assert_close_rel(_np(o["pool"])[:, :P], ref["pool"], STORE_RTOL["bf16"], fp32_atol(host["kv"], nt), "pool")
    assert_close_rel(_np(o["poolI"])[:, :P], ref["poolI"], STORE_RTOL["bf16"], fp32_atol(host["kI"], nt), "poolI")
    assert_close_rel(_np(o["kv_rot"]), ref["kv_rot"], STORE_RTOL["bf16"], fp32_atol(host["kv"], 2), "kv_rot")
    _check_layer_idx_and_out(w, host, o, ref, rows, rel_key_err=STORE_RTOL["bf16"])


def test_hca_prefill_layer_bf16(lib):
    w = synth.WORKLOADS["hca_prefill_bf16"]
    host, o = _run_layer(lib, w)
    rows = [(0, s) for s in sample_rows(w.S, 256, 64)]
    ref = O.hca_layer(host["q"], host["kv"], host["z"], host["bias"], host["sink"], host["pos"], rows=rows,
                      store="bf16", **_oracle_kw(w))
    assert_close_rel(_np(o["pool"]), ref["pool"], STORE_RTOL["bf16"], fp32_atol(host["kv"], w.m), "pool")
    gkv = _np(o["kv_rot"])
    assert_close_rel(gkv[:, ::97], ref["kv_rot"][:, ::97], STORE_RTOL["bf16"], fp32_atol(host["kv"], 2), "kv_rot")
    gout = _np(o["out"])
    for b, s in rows:
        assert_max_abs(gout[b, s], ref["out"][b, s], ATTN_TOL["bf16"], f"out row {s}")


def test_dsa_prefill_layer_bf16(lib):
    w = synth.WORKLOADS["dsa_prefill_bf16"]
    host, o = _run_layer(lib, w)
    rows = [(0, s) for s in sample_rows(w.S, 160, 48)]
    ref = O.csa_layer(host["q"], host["kv"], None, None, host["qI"], host["wI"], host["kI"], None, None,
                      host["sink"], host["pos"], overlap=0, topk=w.topk, store="bf16", rows=rows,
                      **_oracle_kw(w))
    assert_close_rel(_np(o["pool"]), ref["pool"], STORE_RTOL["bf16"], fp32_atol(host["kv"], 2), "pool")
    # m = 1: the indexer pool is the key stream itself
    np.testing.assert_array_equal(_np(o["poolI"]), host["kI"])
    _check_layer_idx_and_out(w, host, o, ref, rows, rel_key_err=STORE_RTOL["bf16"])


# ------------------------------------------------------------------ kernel-level tests
def _cache(w, gains=None):
    sp = synth.cache_specs(w, gains)
    rows = w.win_ring if w.win_ring else w.S
    c = {"pool": sp["pool"].full().reshape(w.B, w.P_cap, w.D),
         "win": sp["win"].full().reshape(w.B, rows, w.D)}
    if "poolI" in sp:
        c["poolI"] = sp["poolI"].full().reshape(w.B, w.P_cap, w.cI)
    return c


def _query_inputs(w, gains=None):
    specs = synth.tensor_specs(w, gains)
    x = {k: synth.reshape(w, k, specs[k].full()) for k in ("q", "sink", "qI", "wI") if k in specs}
    x["q_index"], x["qpos"] = synth.positions(w)
    return x


@pytest.mark.parametrize("name", ["tiny_csa_f32", "csa_prefill_bf16", "csa_decode_bf16", "dsa_prefill_bf16"])
def test_indexer_topk_kernel(lib, name):
    abi, harness = lib
    w = synth.WORKLOADS[name]
    c = _cache(w)
    x = _query_inputs(w)
    params = harness.params_for(w)
    d = harness.to_device(w, {"qI": x["qI"], "wI": x["wI"], "poolI": c["poolI"], "q_index": x["q_index"]})
    idx = torch.empty((w.B, w.Sq, w.topk), dtype=torch.int32, device="cuda")
    ws = torch.empty(max(abi.dsv4_workspace_bytes(params), 256), dtype=torch.uint8, device="cuda")
    abi.dsv4_indexer_topk(params, d["qI"], d["wI"], d["poolI"], d["q_index"], idx, ws)
    torch.cuda.synchronize()
    g = _np(idx)
    rows = [(b, s) for b in range(w.B) for s in (sample_rows(w.Sq, 384, 64) if w.Sq > 1 else [0])]
    excused, stats = 0, {}
    for b, s in rows:
        t = int(x["q_index"][b, s])
        vis = O.visible_entries(t, w.m, w.P_cap)
        sc = O.indexer_scores_row(x["qI"][b, s], x["wI"][b, s], c["poolI"][b], vis)
        err = score_error_bound(x["qI"][b, s], x["wI"][b, s], c["poolI"][b][:vis], 0.0)
        excused += check_topk_row(g[b, s], sc, w.topk, err, stats=stats)
    report(f"indexer_topk {name}", stats)
    assert excused <= max(2, len(rows) // 50), f"{excused} near-tie swaps in {len(rows)} rows"


@pytest.mark.parametrize("name,gains,use_idx", [
    ("tiny_csa_f32", None, True), ("tiny_csa_f32", {"q": 64.0}, True), ("tiny_csa_f32", None, False),
    ("csa_prefill_bf16", None, True), ("csa_prefill_bf16", {"q": 256.0}, True),
    ("hca_prefill_bf16", {"q": 128.0}, False), ("csa_decode_bf16", {"q": 256.0}, True),
    ("dsa_prefill_bf16", {"q": 256.0}, True)])
def test_sparse_attention_kernel(lib, name, gains, use_idx):
    abi, harness = lib
    w = synth.WORKLOADS[name]
    c = _cache(w, gains)
    x = _query_inputs(w, gains)
    idx = synth.strided_selection(w, x["q_index"]) if use_idx else None
    params = harness.params_for(w)
    d = harness.to_device(w, {"q": x["q"], "win": c["win"], "pool": c["pool"], "sink": x["sink"],
                              "qpos": x["qpos"], "q_index": x["q_index"]})
    didx = torch.from_numpy(idx).cuda() if use_idx else None
    out = torch.empty((w.B, w.Sq, w.H, w.dv), dtype=harness.torch_dtype(w), device="cuda")
    ws = torch.empty(max(abi.dsv4_workspace_bytes(params), 256), dtype=torch.uint8, device="cuda")
    abi.dsv4_sparse_mqa_attn(params, d["q"], d["win"], d["pool"], didx, d["sink"], d["qpos"], d["q_index"], out, ws)
    abi.dsv4_device_check()
    rows = [(b, s) for b in range(w.B) for s in (sample_rows(w.Sq, 192, 32) if w.Sq > 1 else [0])]
    ref = O.sparse_mqa_attention(x["q"], c["win"], c["pool"], idx, x["sink"], x["qpos"], x["q_index"],
                                 n_win=w.n_win, m=w.m, scale=w.scale, dv=w.dv, R=w.R, theta=w.theta, rope_q=True,
                                 rotate_out=w.rotate_out, win_ring=w.win_ring, P_cap=w.P_cap, rows=rows)
    g = _np(out)
    for b, s in rows:
        assert_max_abs(g[b, s], ref[b, s], ATTN_TOL[w.dtype], f"{name} row {(b, s)}")


@pytest.mark.parametrize("B,with_ws,S", [(3, True, 20000), (3, False, 20000), (40, True, 20000), (3, True, 600)])
def test_decode_attention_key_splits(lib, B, with_ws, S):
    """Few queries: the keys of each query are split over CTAs and merged (or not, without a
    workspace).  The split count comes from the sizes (window + top-k keys); with S=600 the
    caches hold at most 150 entries, so most of the 9 splits of a query are empty."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_decode_bf16"].replace(B=B, S=S, P_cap=5000, topk=1024, qindex_spread=500)
    c = _cache(w, {"q": 256.0})
    x = _query_inputs(w, {"q": 256.0})
    idx = synth.strided_selection(w, x["q_index"])
    params = harness.params_for(w)
    d = harness.to_device(w, {"q": x["q"], "win": c["win"], "pool": c["pool"], "sink": x["sink"],
                              "qpos": x["qpos"], "q_index": x["q_index"]})
    out = torch.empty((w.B, 1, w.H, w.dv), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(abi.dsv4_workspace_bytes(params), 256), dtype=torch.uint8, device="cuda") if with_ws else None
    abi.dsv4_sparse_mqa_attn(params, d["q"], d["win"], d["pool"], torch.from_numpy(idx).cuda(), d["sink"],
                             d["qpos"], d["q_index"], out, ws)
    abi.dsv4_device_check()
    rows = [(b, 0) for b in range(w.B)]
    ref = O.sparse_mqa_attention(x["q"], c["win"], c["pool"], idx, x["sink"], x["qpos"], x["q_index"],
                                 n_win=w.n_win, m=w.m, scale=w.scale, dv=w.dv, R=w.R, theta=w.theta, rope_q=True,
                                 rotate_out=w.rotate_out, win_ring=w.win_ring, P_cap=w.P_cap, rows=rows)
    g = _np(out)
    for b, s in rows:
        assert_max_abs(g[b, s], ref[b, s], ATTN_TOL["bf16"], f"decode row {b}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("overlap,m", [(1, 4), (0, 8), (0, 1)])
def test_compress_kernel_ragged(lib, dtype, overlap, m):
    """S not a multiple of m, B = 2, pool capacity above S/m, positions offset."""
    abi, harness = lib
    w = synth.WORKLOADS["tiny_csa_f32"].replace(dtype=dtype, B=2, S=203, Sq=203, P_cap=260, m=m, overlap=overlap)
    host = synth.make_inputs(w)
    if m == 1:
        host.pop("z", None), host.pop("bias", None)
    host["pos"] = host["pos"] + 1000
    params = harness.params_for(w)
    d = harness.to_device(w, host)
    pool = torch.zeros((w.B, w.P_cap, w.D), dtype=harness.torch_dtype(w), device="cuda")
    xr = torch.zeros((w.B, w.S, w.D), dtype=harness.torch_dtype(w), device="cuda")
    abi.dsv4_compress_kv(params, w.D, d["kv"], d.get("z"), d.get("bias"), d["pos"], 1, pool, xr)
    torch.cuda.synchronize()
    P = w.S // m
    ref = O.compress(host["kv"], host.get("z"), host.get("bias"), host["pos"], m=m, overlap=overlap,
                     apply_rope=True, R=w.R, theta=w.theta)
    tol = STORE_RTOL[dtype]
    nt = 2 * m if overlap else m
    assert_close_rel(_np(pool)[:, :P], ref, tol, fp32_atol(host["kv"], nt), "pool")
    assert np.all(_np(pool)[:, P:] == 0), "entries past S/m must be left untouched"
    assert_close_rel(_np(xr), O.rope_rotate(host["kv"], host["pos"], w.R, w.theta), tol,
                     fp32_atol(host["kv"], 2), "x_rot")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_ragged_layers(lib, dtype):
    """A CSA layer with B=2, ragged S, a window of 5, top-k larger than early pools, and an HCA layer."""
    abi, harness = lib
    base = synth.WORKLOADS["tiny_csa_f32"].replace(dtype=dtype, B=2, S=150, Sq=150, H=16, D=64, R=32, dv=64,
                                                 n_win=5, m=4, overlap=1, nI=2, cI=32, topk=20, P_cap=40)
    for w in (base, base.replace(kind="hca", m=16, overlap=0, nI=0, cI=0, topk=0, P_cap=9)):
        host, o = _run_layer(lib, w)
        kw = _oracle_kw(w)
        if w.kind == "csa":
            ref = O.csa_layer(host["q"], host["kv"], host["z"], host["bias"], host["qI"], host["wI"], host["kI"],
                              host["zI"], host["biasI"], host["sink"], host["pos"], overlap=1, topk=w.topk,
                              store=STORE[dtype], **kw)
            rows = [(b, s) for b in range(w.B) for s in range(w.S)]
            _check_layer_idx_and_out(w, host, o, ref, rows, rel_key_err=STORE_RTOL[dtype] * 2)
        else:
            ref = O.hca_layer(host["q"], host["kv"], host["z"], host["bias"], host["sink"], host["pos"],
                              store=STORE[dtype], **kw)
            assert_max_abs(_np(o["out"]), ref["out"], ATTN_TOL[dtype], "hca out")


def test_empty_batch_is_a_noop(lib):
    abi, harness = lib
    w = synth.WORKLOADS["tiny_csa_f32"]
    p = harness.params_for(w, B=0)
    t = torch.zeros(16, device="cuda")
    abi.dsv4_sparse_mqa_attn(p, t, t, t, None, t, t, None, t)
    abi.dsv4_compress_kv(p, w.D, t, None, None, t, 1, t, None)
    torch.cuda.synchronize()
    assert torch.all(t == 0)


def test_layer_is_deterministic(lib):
    w = synth.WORKLOADS["csa_prefill_bf16"].replace(S=2048, Sq=2048, P_cap=512)
    abi, harness = lib
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o1 = harness.make_outputs(w, params)
    o2 = harness.make_outputs(w, params)
    harness.step(w, params, x, o1)
    harness.step(w, params, x, o2)
    torch.cuda.synchronize()
    assert torch.equal(o1["idx"], o2["idx"])
    assert torch.equal(o1["out"].view(torch.int16), o2["out"].view(torch.int16))


@pytest.mark.parametrize("name,gains", [("tiny_csa_f32", None), ("csa_prefill_bf16", None),
                                        ("csa_prefill_bf16", {"q": 256.0})])
def test_sliding_window_only_attention(lib, name, gains):
    """`sliding_attention` layers ("DeepSeek-V4", layer types): the window branch alone — no
    pool, no index lists (pool NULL, P_cap 0) — over rows already rotated at their positions."""
    abi, harness = lib
    w0 = synth.WORKLOADS[name]
    w = w0.replace(S=min(w0.S, 1024), Sq=min(w0.S, 1024), P_cap=0, topk=0, nI=0)
    specs = synth.tensor_specs(w, gains)
    q = synth.reshape(w, "q", specs["q"].full())
    kv = synth.reshape(w, "kv", specs["kv"].full())
    sink = specs["sink"].full()
    qi, qp = synth.positions(w)
    params = harness.params_for(w)
    d = harness.to_device(w, {"q": q, "kv": kv, "sink": sink, "qpos": qp, "q_index": qi})
    out = torch.empty((w.B, w.Sq, w.H, w.dv), dtype=harness.torch_dtype(w), device="cuda")
    ws = torch.empty(max(abi.dsv4_workspace_bytes(params), 256), dtype=torch.uint8, device="cuda")
    abi.dsv4_sparse_mqa_attn(params, d["q"], d["kv"], None, None, d["sink"], d["qpos"], d["q_index"], out, ws)
    abi.dsv4_device_check()
    rows = [(0, s) for s in sample_rows(w.Sq, 128, 16)]
    ref = O.sparse_mqa_attention(q, kv, np.zeros((w.B, 0, w.D)), None, sink, qp, qi, n_win=w.n_win, m=w.m,
                                 scale=w.scale, dv=w.dv, R=w.R, theta=w.theta, rope_q=True,
                                 rotate_out=w.rotate_out, P_cap=0, rows=rows)
    g = _np(out)
    for b, s in rows:
        assert_max_abs(g[b, s], ref[b, s], ATTN_TOL[w.dtype], f"{name} window-only row {(b, s)}")


def test_bench_step_path_csa_prefill(lib):
    """The exact path bench.py times (harness.step_parts: the compressor, dsv4_indexer_scores
    and dsv4_topk_select, the attention) at the full CSA prefill size, on sampled rows."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_prefill_bf16"]
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o = harness.make_outputs(w, params, scores=True)
    harness.step_parts(w, params, x, o)
    abi.dsv4_device_check()
    rows = [(0, s) for s in sample_rows(w.S, 192, 32)]
    ref = O.csa_layer(host["q"], host["kv"], host["z"], host["bias"], host["qI"], host["wI"], host["kI"],
                      host["zI"], host["biasI"], host["sink"], host["pos"], overlap=w.overlap, topk=w.topk,
                      store="bf16", rows=rows, **_oracle_kw(w))
    _check_layer_idx_and_out(w, host, o, ref, rows, rel_key_err=STORE_RTOL["bf16"])


def test_bench_step_path_csa_decode(lib):
    """The exact decode path bench.py times, at the full decode size (64 sequences, pool
    32768, top-2048): top-k rows against the oracle's scores, attention rows whose
    selection matches the oracle's."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_decode_bf16"]
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o = harness.make_outputs(w, params, scores=True)
    harness.step_parts(w, params, x, o)
    abi.dsv4_device_check()
    gidx, gout = _np(o["idx"]), _np(o["out"])
    stats = {}
    for b in range(0, w.B, 9):
        t = int(host["q_index"][b, 0])
        vis = O.visible_entries(t, w.m, w.P_cap)
        sc = O.indexer_scores_row(host["qI"][b, 0], host["wI"][b, 0], host["poolI"][b], vis)
        err = score_error_bound(host["qI"][b, 0], host["wI"][b, 0], host["poolI"][b][:vis], 0.0)
        check_topk_row(gidx[b, 0], sc, w.topk, err, stats=stats)
        # the GPU's selection (equal to the oracle's, or differing only at excused near ties)
        sel = gidx[b:b + 1, :1].astype(np.int64)
        ref = O.sparse_mqa_attention(host["q"][b:b + 1], host["win"][b:b + 1], host["pool"][b:b + 1], sel,
                                     host["sink"], host["qpos"][b:b + 1], host["q_index"][b:b + 1],
                                     n_win=w.n_win, m=w.m, scale=w.scale, dv=w.dv, R=w.R, theta=w.theta,
                                     rope_q=True, rotate_out=w.rotate_out, win_ring=w.win_ring, P_cap=w.P_cap)
        assert_max_abs(gout[b, 0], ref[0, 0], ATTN_TOL[w.dtype], f"decode row {b}")
    report("csa_decode_bf16 bench path", stats)


def test_bench_step_path_swa_prefill(lib):
    """The sliding-window layer bench.py times, at full size (B=1, S=8192, 64 heads, window
    128): RoPE of the K=V rows with no pool (rotated rows within one storage ulp of the
    oracle's), then attention over the window alone (sampled rows within the attention
    tolerance of the oracle's sliding layer, which reads the same bf16-stored rows)."""
    abi, harness = lib
    w = synth.WORKLOADS["swa_prefill_bf16"]
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o = harness.make_outputs(w, params, scores=True)
    assert "pool" not in o and "idx" not in o
    harness.step_parts(w, params, x, o)
    abi.dsv4_device_check()
    rot = O.rope_rotate(host["kv"], host["pos"], w.R, w.theta)
    assert_close_rel(_np(o["kv_rot"]), rot, STORE_RTOL["bf16"], fp32_atol(host["kv"], 4), "rotated K=V rows")
    rows = [(0, s) for s in sample_rows(w.S, 192, 32)]
    ref = O.sliding_layer(host["q"], host["kv"], host["sink"], host["pos"], n_win=w.n_win, scale=w.scale,
                          dv=w.dv, R=w.R, theta=w.theta, rotate_out=w.rotate_out, rows=rows, store="bf16")
    g = _np(o["out"])
    for b, s in rows:
        assert_max_abs(g[b, s], ref["out"][b, s], ATTN_TOL["bf16"], f"window-only row {s}")


def test_index_checks_report_bad_lists(lib):
    """With the index checks on, dsv4_sparse_mqa_attn validates its index lists on the device:
    a valid list passes; a duplicated entry, an entry that is not yet visible and an entry
    below -1 each make dsv4_device_check report DSV4_ERR_DEVICE_CHECK (the attention still
    runs, masking what it cannot use, and nothing traps)."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_prefill_bf16"].replace(S=1024, Sq=1024, P_cap=256, topk=64)
    c = _cache(w)
    x = _query_inputs(w)
    idx = synth.strided_selection(w, x["q_index"])
    params = harness.params_for(w)
    d = harness.to_device(w, {"q": x["q"], "win": c["win"], "pool": c["pool"], "sink": x["sink"],
                              "qpos": x["qpos"], "q_index": x["q_index"]})
    out = torch.empty((w.B, w.Sq, w.H, w.dv), dtype=torch.bfloat16, device="cuda")

    def run(lists):
        abi.dsv4_sparse_mqa_attn(params, d["q"], d["win"], d["pool"], torch.from_numpy(lists).cuda(), d["sink"],
                                 d["qpos"], d["q_index"], out)

    abi.dsv4_device_check()  # start from a clear word
    abi.dsv4_set_index_checks(True)
    try:
        assert abi.dsv4_index_checks()
        run(idx)
        abi.dsv4_device_check()
        t = 900                       # vis = 225 entries, 64 selected
        vis = (t + 1) // w.m
        for name, edit in (("duplicate", lambda r: r.__setitem__(1, r[0])),
                           ("not visible", lambda r: r.__setitem__(0, vis)),
                           ("below -1", lambda r: r.__setitem__(2, -5))):
            bad = idx.copy()
            edit(bad[0, t])
            run(bad)
            with pytest.raises(abi.Dsv4Error) as e:
                abi.dsv4_device_check()
            assert e.value.status == 6, name
            abi.dsv4_device_check()   # the word was cleared by the failing check
    finally:
        abi.dsv4_set_index_checks(False)
    assert not abi.dsv4_index_checks()
