"""Device-side plumbing around the C ABI: parameters, buffers and one step of a workload.

A "step" is one pass of the hot path over one batch:
  prefill CSA / DSA: dsv4_csa_layer (compress kv, compress kI, indexer + top-k, attention)
  prefill HCA:       dsv4_hca_layer (compress kv, attention over every visible entry)
  decode:            dsv4_indexer_topk + dsv4_sparse_mqa_attn over a pre-filled cache
  sliding window:    dsv4_compress_kv without a pool (RoPE of the K=V rows) +
                     dsv4_sparse_mqa_attn over the window alone
  decode append:     dsv4_decode_append of one token per sequence to the K=V stream
                     (buffer, window ring, pool) and to the indexer-key stream
  output projection: dsv4_grouped_out_proj of the attention output (o_a_proj per head
                     group, then o_b_proj)
PyTorch only allocates device memory and supplies the stream; every step of the
method runs inside libdsv4.
"""
from __future__ import annotations

import torch

from . import abi


def params_for(w, **over) -> abi.Dsv4Params:
    """dsv4_params of a workload description (``synth.Workload``-like object)."""
    p = abi.Dsv4Params()
    p.B, p.S, p.Sq, p.H, p.D, p.R, p.dv = w.B, w.S, w.Sq, w.H, w.D, w.R, w.dv
    p.n_win, p.win_ring, p.m, p.overlap, p.P_cap = w.n_win, w.win_ring, w.m, w.overlap, w.P_cap
    p.nI, p.cI, p.topk = w.nI, w.cI, w.topk
    p.scale, p.rope_theta = w.scale, w.theta
    p.rope_q, p.rotate_out = 1, w.rotate_out
    p.dtype = abi.BF16 if w.dtype == "bf16" else abi.F32
    for k, v in over.items():
        setattr(p, k, v)
    return p


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


FLOAT_ACT = ("q", "kv", "z", "qI", "kI", "zI", "pool", "poolI", "win", "o", "wa", "wb")  # activation dtype
FLOAT_F32 = ("bias", "biasI", "wI", "sink")                             # always fp32


def to_device(w, host: dict, device="cuda", pin=False) -> dict:
    """Copy host numpy inputs to device tensors of the storage dtypes the ABI expects."""
    dt = torch_dtype(w)
    out = {}
    for k, v in host.items():
        t = torch.from_numpy(v)
        if k in FLOAT_ACT:
            t = t.to(device).to(dt) if (device and not pin) else t.to(dt)
        elif k in FLOAT_F32:
            t = t.to(torch.float32)
        elif k == "q_index":
            t = t.to(torch.int32)
        elif k in ("pos", "qpos"):
            t = t.to(torch.int64)
        if pin:
            t = t.pin_memory()
        out[k] = t.to(device, non_blocking=pin) if device else t
    return out


def append_state(w, device="cuda") -> dict:
    """Decode-cache state of both streams of a workload of kind "append", zero-filled: the
    compressor buffers (Lw rows, their logits and positions), the K=V window ring and the
    two pools."""
    dt = torch_dtype(w)
    lw = 2 * w.m if w.overlap else w.m

    def z(*shape, dtype=dt):
        return torch.zeros(shape, dtype=dtype, device=device)

    return {"buf_x": z(w.B, lw, w.D), "buf_z": z(w.B, lw, w.D), "buf_pos": z(w.B, lw, dtype=torch.int64),
            "bufI_x": z(w.B, lw, w.cI), "bufI_z": z(w.B, lw, w.cI), "bufI_pos": z(w.B, lw, dtype=torch.int64),
            "win": z(w.B, w.win_ring, w.D), "pool": z(w.B, w.P_cap, w.D), "poolI": z(w.B, w.P_cap, w.cI)}


def make_outputs(w, params: abi.Dsv4Params, device="cuda", scores=False) -> dict:
    dt = torch_dtype(w)
    if w.kind == "append":
        return append_state(w, device)
    if w.kind == "outproj":
        T = w.B * w.Sq
        return {"u": torch.empty((T, w.o_groups * w.o_rank), dtype=dt, device=device),
                "out": torch.empty((T, w.hidden), dtype=dt, device=device)}
    o = {"out": torch.empty((w.B, w.Sq, w.H, w.dv), dtype=dt, device=device)}
    if w.kind != "decode":
        if w.P_cap > 0:
            o["pool"] = torch.empty((w.B, w.P_cap, w.D), dtype=dt, device=device)
        o["kv_rot"] = torch.empty((w.B, w.S, w.D), dtype=dt, device=device)
    if w.nI > 0:
        if w.kind != "decode":
            o["poolI"] = torch.empty((w.B, w.P_cap, w.cI), dtype=dt, device=device)
        o["idx"] = torch.empty((w.B, w.Sq, w.topk), dtype=torch.int32, device=device)
    ws = abi.dsv4_workspace_bytes(params)
    o["workspace"] = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
    if w.nI > 0 and scores:
        o["scores"] = torch.empty((w.B * w.Sq, w.P_cap), dtype=torch.float32, device=device)
    return o


_SIDE_STREAMS: dict = {}


def _side_stream(device) -> "torch.cuda.Stream":
    if device not in _SIDE_STREAMS:
        _SIDE_STREAMS[device] = torch.cuda.Stream(device=device)
    return _SIDE_STREAMS[device]


def append_token(w, params, x: dict, o: dict, k: int, stream=None) -> None:
    """Append history token k (rows x["kv"][k], x["kI"][k], ...) to every sequence's cache:
    the K=V stream (rotated window row; entry pooled and rotated when the token closes a
    block) on ``stream`` and, concurrently, the indexer-key stream (no RoPE, no window) on
    a side stream that forks from and joins back into ``stream``: the two caches share no
    memory, and each launch is latency-bound."""
    main = stream if stream is not None else torch.cuda.current_stream()
    side = _side_stream(main.device)
    fork = torch.cuda.Event()
    fork.record(main)
    side.wait_event(fork)
    abi.dsv4_decode_append(params, w.D, x["kv"][k], x["z"][k], x["bias"], x["pos_hist"][k], x["t_hist"][k],
                           o["buf_x"], o["buf_z"], o["buf_pos"], 1, o["win"], o["pool"], stream=main)
    abi.dsv4_decode_append(params, w.cI, x["kI"][k], x["zI"][k], x["biasI"], x["pos_hist"][k], x["t_hist"][k],
                           o["bufI_x"], o["bufI_z"], o["bufI_pos"], 0, None, o["poolI"], stream=side)
    join = torch.cuda.Event()
    join.record(side)
    main.wait_event(join)


def append_prefill(w, params, x: dict, o: dict, stream=None) -> None:
    """Bring the cache to the state just before the step's token: append the Lw-1 tokens
    before it, so that the buffers hold every token that the step's pooling reads."""
    for k in range(x["kv"].shape[0] - 1):
        append_token(w, params, x, o, k, stream)


def step(w, params, x: dict, o: dict, stream=None) -> None:
    """Enqueue one step of the workload's hot path (see module docstring)."""
    if w.kind == "append":
        append_token(w, params, x, o, x["kv"].shape[0] - 1, stream)
        return
    if w.kind == "outproj":
        abi.dsv4_grouped_out_proj(params, w.B * w.Sq, w.o_groups, w.o_rank, w.hidden, x["o"], x["wa"], x["wb"],
                                  o["u"], o["out"], stream=stream)
        return
    ws = o["workspace"]
    if w.kind in ("csa", "dsa"):
        abi.dsv4_csa_layer(params, x["q"], x["kv"], x.get("z"), x.get("bias"), x["qI"], x["wI"], x["kI"],
                           x.get("zI"), x.get("biasI"), x["sink"], x["pos"], o["out"], o["pool"], o["poolI"],
                           o["kv_rot"], o["idx"], ws, stream=stream)
    elif w.kind == "hca":
        abi.dsv4_hca_layer(params, x["q"], x["kv"], x.get("z"), x.get("bias"), x["sink"], x["pos"], o["out"],
                           o["pool"], o["kv_rot"], ws, stream=stream)
    elif w.kind == "decode":
        abi.dsv4_indexer_topk(params, x["qI"], x["wI"], x["poolI"], x["q_index"], o["idx"], ws, stream=stream)
        abi.dsv4_sparse_mqa_attn(params, x["q"], x["win"], x["pool"], o["idx"], x["sink"], x["qpos"],
                                 x["q_index"], o["out"], ws, stream=stream)
    elif w.kind == "swa":
        step_parts(w, params, x, o, stream)
    else:
        raise ValueError(w.kind)


PARTS = ("append", "compress", "indexer_topk", "indexer_scores", "topk", "attention", "out_proj")


def step_input_keys(w) -> list:
    """The per-step activations a step reads (what a serving loop copies in every step); the
    layer weights (compressor bias, sink) and the decode cache stay resident on the device."""
    if w.kind == "decode":
        return ["q", "qI", "wI", "q_index", "qpos"]
    if w.kind == "append":
        return ["kv", "z", "kI", "zI", "pos_hist", "t_hist"]
    if w.kind == "outproj":
        return ["o"]
    keys = ["q", "kv", "z", "pos"]
    if w.nI > 0:
        keys += ["qI", "wI", "kI", "zI"]
    return keys


def selects_in_attention(w) -> bool:
    """CSA prefill whose score rows are short enough for the attention kernel to select each
    query's index list itself (dsv4_sparse_mqa_attn_scores: bf16, P_cap <= 2048, topk <= 512)."""
    return w.kind == "csa" and w.dtype == "bf16" and 0 < w.P_cap <= 2048 and 0 < w.topk <= 512


def step_parts(w, params, x: dict, o: dict, stream=None, events=None) -> None:
    """The same step as ``step`` issued entry point by entry point: for prefill the indexer
    scores (dsv4_indexer_scores into ``o["scores"]``), then either the selection inside the
    attention (dsv4_sparse_mqa_attn_scores, as dsv4_csa_layer does when the rows are short) or
    dsv4_topk_select and dsv4_sparse_mqa_attn; for decode dsv4_indexer_topk, whose one kernel
    scores and selects.  The same kernels on the same data as ``step``.  ``events`` maps names
    of ``PARTS`` to (start, end) CUDA event pairs recorded on ``stream`` around that part."""
    ws = o.get("workspace")

    def mark(name, k):
        if events is not None and name in events:
            events[name][k].record(stream)

    if w.kind == "append":
        mark("append", 0)
        step(w, params, x, o, stream)
        mark("append", 1)
        return
    if w.kind == "outproj":
        mark("out_proj", 0)
        step(w, params, x, o, stream)
        mark("out_proj", 1)
        return
    if w.kind in ("csa", "dsa", "hca", "swa"):
        mark("compress", 0)
        abi.dsv4_compress_kv(params, w.D, x["kv"], x.get("z"), x.get("bias"), x["pos"], 1, o.get("pool"),
                             o["kv_rot"], stream=stream)
        if w.kind in ("csa", "dsa"):
            abi.dsv4_compress_kv(params, w.cI, x["kI"], x.get("zI"), x.get("biasI"), None, 0, o["poolI"], None,
                                 stream=stream)
        mark("compress", 1)
    if w.kind == "decode":
        # one query per sequence: dsv4_indexer_topk scores and selects in one kernel
        mark("indexer_topk", 0)
        abi.dsv4_indexer_topk(params, x["qI"], x["wI"], x["poolI"], x["q_index"], o["idx"], ws, stream=stream)
        mark("indexer_topk", 1)
    elif w.nI > 0:
        poolI = o["poolI"]
        q_index = None
        mark("indexer_scores", 0)
        abi.dsv4_indexer_scores(params, x["qI"], x["wI"], poolI, q_index, o["scores"], stream=stream)
        mark("indexer_scores", 1)
        if not selects_in_attention(w):
            mark("topk", 0)
            abi.dsv4_topk_select(params, o["scores"], q_index, o["idx"], stream=stream)
            mark("topk", 1)
    mark("attention", 0)
    if w.kind == "decode":
        abi.dsv4_sparse_mqa_attn(params, x["q"], x["win"], x["pool"], o["idx"], x["sink"], x["qpos"],
                                 x["q_index"], o["out"], ws, stream=stream)
    elif w.nI > 0 and selects_in_attention(w):
        abi.dsv4_sparse_mqa_attn_scores(params, x["q"], o["kv_rot"], o["pool"], o["scores"], x["sink"], x["pos"],
                                        None, o["idx"], o["out"], ws, stream=stream)
    else:
        abi.dsv4_sparse_mqa_attn(params, x["q"], o["kv_rot"], o.get("pool"), o.get("idx"), x["sink"], x["pos"],
                                 None, o["out"], ws, stream=stream)
    mark("attention", 1)
