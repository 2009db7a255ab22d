"""Decode-cache append (dsv4_decode_append) against the oracle and against the prefill compressor.

Two sequences append the tokens of a synthetic prefix one launch at a time (the second starts
37 launches later, so the batch mixes cache indices and skipped sequences).  Afterwards:
  * the pool equals the oracle's compression of the prefix (readings R1-R3) within one
    storage ulp plus the fp32 accumulation bound, and the window ring holds the last rows
    rotated at their positions;
  * the pool and the window ring are bit-identical to what dsv4_compress_kv writes for the
    same rows (one pooling routine, same arithmetic).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from oracle import dsv4_oracle as O
from parity_util import assert_close_rel

pytestmark = pytest.mark.gpu

STORE_RTOL = {"f32": 2.0 ** -23, "bf16": 2.0 ** -7}
U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def lib():
    from sparse_long_context_csa_b200 import abi, harness
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    return abi, harness


@pytest.mark.parametrize("name,stream", [("tiny_csa_f32", "kv"), ("tiny_csa_f32", "kI"),
                                         ("csa_prefill_bf16", "kv"), ("csa_prefill_bf16", "kI"),
                                         ("hca_prefill_bf16", "kv")])
def test_decode_append_matches_prefill_compression(lib, name, stream):
    abi, harness = lib
    w0 = synth.WORKLOADS[name]
    S, lag, ring = 300, 37, 64
    w = w0.replace(B=2, S=S, Sq=S, P_cap=S // w0.m)
    host = synth.make_inputs(w)
    rope = stream == "kv"
    key = {"kv": ("kv", "z", "bias"), "kI": ("kI", "zI", "biasI")}[stream]
    x, z, bias = (host.get(k) for k in key)
    c = x.shape[-1]
    lw = 2 * w.m if w.overlap else w.m
    params = harness.params_for(w, win_ring=ring)
    dt = harness.torch_dtype(w)
    dev = "cuda"
    xd = torch.from_numpy(x).to(dev, dt)
    zd = torch.from_numpy(z).to(dev, dt) if z is not None else None
    bd = torch.from_numpy(bias).to(dev, torch.float32).contiguous() if bias is not None else None
    posd = torch.from_numpy(host["pos"]).to(dev)
    # per-launch inputs: sequence b appends token step - b*lag (or is skipped)
    steps = S + lag
    tt = np.full((steps, 4), -1, dtype=np.int32)      # rows padded to 16 bytes
    for st in range(steps):
        for b in range(2):
            t = st - b * lag
            tt[st, b] = t if 0 <= t < S else -1
    ti = torch.from_numpy(np.clip(tt[:, :2], 0, S - 1)).to(dev).long()
    bidx = torch.arange(2, device=dev)
    x_st = xd[bidx[None, :], ti].contiguous()             # [steps, B, c]
    z_st = zd[bidx[None, :], ti].contiguous() if zd is not None else None
    p_st = posd[bidx[None, :], ti].contiguous()           # [steps, B]
    t_st = torch.from_numpy(tt).to(dev)
    buf_x = torch.zeros((2, lw, c), dtype=dt, device=dev)
    buf_z = torch.zeros((2, lw, c), dtype=dt, device=dev) if zd is not None else None
    buf_p = torch.zeros((2, lw), dtype=torch.int64, device=dev)
    win = torch.zeros((2, ring, c), dtype=dt, device=dev) if rope else None
    pool = torch.full((2, w.P_cap, c), float("nan"), dtype=dt, device=dev)
    for st in range(steps):
        abi.dsv4_decode_append(params, c, x_st[st], z_st[st] if z_st is not None else None, bd, p_st[st],
                               t_st[st], buf_x, buf_z, buf_p, int(rope), win, pool)
    abi.dsv4_device_check()

    P = S // w.m
    ref = O.compress(x, z, bias, host["pos"], m=w.m, overlap=w.overlap, apply_rope=rope, R=w.R, theta=w.theta)
    g = pool.float().cpu().numpy()
    nt = lw
    assert_close_rel(g[:, :P], ref, STORE_RTOL[w.dtype], (nt + 8) * U32 * float(np.abs(x).max()), "appended pool")

    # the prefill compressor on the same rows: the same bits
    pool_b = torch.zeros_like(pool)
    xrot_b = torch.zeros_like(xd) if rope else None
    abi.dsv4_compress_kv(params, c, xd, zd, bd, posd if rope else None, int(rope), pool_b, xrot_b)
    abi.dsv4_device_check()
    assert torch.equal(pool[:, :P], pool_b[:, :P]), "appended entries differ from dsv4_compress_kv's"
    if rope:
        last = torch.arange(S - ring, S, device=dev)
        assert torch.equal(win[:, last % ring], xrot_b[:, last]), "window ring differs from the rotated rows"
        rot = O.rope_rotate(x, host["pos"], w.R, w.theta)
        gw = win.float().cpu().numpy()
        for j in range(S - ring, S):
            assert_close_rel(gw[:, j % ring], rot[:, j], STORE_RTOL[w.dtype], 4 * U32 * float(np.abs(x).max()),
                             f"window row {j}")


def test_bench_step_path_decode_append(lib):
    """The decode-cache append bench.py times, at full size (64 sequences, pool 32768, window
    ring 128, K=V and indexer-key streams): the Lw-1 earlier tokens and then the step's token
    are appended to zeroed caches on both sides.  Every sequence's window slot holds its
    rotated token; every entry closed on the way matches the oracle's; the buffered positions
    are exact; repeating the step changes no bit."""
    abi, harness = lib
    w = synth.WORKLOADS["csa_decode_append_bf16"]
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o = harness.make_outputs(w, params)
    harness.append_prefill(w, params, x, o)
    harness.step_parts(w, params, x, o)
    abi.dsv4_device_check()
    lw = host["kv"].shape[0]
    t_last = host["t_hist"][-1].astype(np.int64)
    bidx = torch.arange(w.B, device="cuda")
    wslot = torch.from_numpy(t_last % w.win_ring).cuda()
    closes = [(k, b) for k in range(lw) for b in range(w.B) if (int(host["t_hist"][k, b]) + 1) % w.m == 0]
    eb = torch.tensor([b for _, b in closes], device="cuda")
    ew = torch.tensor([(int(host["t_hist"][k, b]) + 1) // w.m - 1 for k, b in closes], device="cuda")
    before = (o["win"][bidx, wslot].clone(), o["buf_x"].clone(), o["buf_pos"].clone(), o["pool"][eb, ew].clone(),
              o["poolI"][eb, ew].clone())
    harness.step(w, params, x, o)   # the timed step once more: the same slots, the same bits
    abi.dsv4_device_check()
    after = (o["win"][bidx, wslot], o["buf_x"], o["buf_pos"], o["pool"][eb, ew], o["poolI"][eb, ew])
    for u, v in zip(before, after):
        assert torch.equal(u, v), "repeating the append changed the cache"

    g_win = before[0].float().cpu().numpy()
    g_pos = before[2].cpu().numpy()
    g_pool = {(k, b): r for (k, b), r in zip(closes, before[3].float().cpu().numpy())}
    g_poolI = {(k, b): r for (k, b), r in zip(closes, before[4].float().cpu().numpy())}
    kw = dict(m=w.m, overlap=w.overlap, R=w.R, theta=w.theta)
    for b in range(w.B):
        kvc = O.new_decode_cache(w.D, m=w.m, overlap=w.overlap, P_cap=w.P_cap, win_ring=w.win_ring)
        kic = O.new_decode_cache(w.cI, m=w.m, overlap=w.overlap, P_cap=w.P_cap)
        for k in range(lw):
            t, pos = int(host["t_hist"][k, b]), int(host["pos_hist"][k, b])
            O.decode_append(kvc, host["kv"][k, b], host["z"][k, b], pos, t, bias=host["bias"], apply_rope=True, **kw)
            O.decode_append(kic, host["kI"][k, b], host["zI"][k, b], pos, t, bias=host["biasI"], apply_rope=False,
                            **kw)
            if (t + 1) % w.m == 0:
                e = (t + 1) // w.m - 1
                assert_close_rel(g_pool[(k, b)], kvc["pool"][e], STORE_RTOL["bf16"],
                                 (lw + 8) * U32 * float(np.abs(host["kv"]).max()), f"K=V entry {e} of seq {b}")
                assert_close_rel(g_poolI[(k, b)], kic["pool"][e], STORE_RTOL["bf16"],
                                 (lw + 8) * U32 * float(np.abs(host["kI"]).max()), f"indexer entry {e} of seq {b}")
        assert_close_rel(g_win[b], kvc["win"][t_last[b] % w.win_ring], STORE_RTOL["bf16"],
                         4 * U32 * float(np.abs(host["kv"]).max()), f"window row of seq {b}")
        np.testing.assert_array_equal(g_pos[b], kvc["pos"])
