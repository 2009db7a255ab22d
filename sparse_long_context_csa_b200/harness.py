"""Device-side plumbing around the C ABI: parameters, buffers and one step of a workload.

A "step" is one pass of the hot path over one batch:
  prefill CSA / DSA: dsv4_csa_layer (compress kv, compress kI, indexer + top-k, attention)
  prefill HCA:       dsv4_hca_layer (compress kv, attention over every visible entry)
  decode:            dsv4_indexer_topk + dsv4_sparse_mqa_attn over a pre-filled cache
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


FLOAT_ACT = ("q", "kv", "z", "qI", "kI", "zI", "pool", "poolI", "win")  # stored in the activation dtype
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


def make_outputs(w, params: abi.Dsv4Params, device="cuda", scores=False) -> dict:
    dt = torch_dtype(w)
    o = {"out": torch.empty((w.B, w.Sq, w.H, w.dv), dtype=dt, device=device)}
    if w.kind != "decode":
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


def step(w, params, x: dict, o: dict, stream=None) -> None:
    """Enqueue one step of the workload's hot path (see module docstring)."""
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
    else:
        raise ValueError(w.kind)


PARTS = ("compress", "indexer_scores", "topk", "attention")


def step_parts(w, params, x: dict, o: dict, stream=None, events=None) -> None:
    """The same step as ``step`` issued entry point by entry point, the indexer as its two
    halves (dsv4_indexer_scores into ``o["scores"]``, then dsv4_topk_select): the same
    kernels on the same data.  ``events`` maps names of ``PARTS`` to (start, end) CUDA
    event pairs recorded on ``stream`` around that part."""
    ws = o["workspace"]

    def mark(name, k):
        if events is not None and name in events:
            events[name][k].record(stream)

    if w.kind in ("csa", "dsa", "hca"):
        mark("compress", 0)
        abi.dsv4_compress_kv(params, w.D, x["kv"], x.get("z"), x.get("bias"), x["pos"], 1, o["pool"],
                             o["kv_rot"], stream=stream)
        if w.kind != "hca":
            abi.dsv4_compress_kv(params, w.cI, x["kI"], x.get("zI"), x.get("biasI"), None, 0, o["poolI"], None,
                                 stream=stream)
        mark("compress", 1)
    if w.nI > 0:
        poolI = o["poolI"] if w.kind != "decode" else x["poolI"]
        q_index = x["q_index"] if w.kind == "decode" else None
        mark("indexer_scores", 0)
        abi.dsv4_indexer_scores(params, x["qI"], x["wI"], poolI, q_index, o["scores"], stream=stream)
        mark("indexer_scores", 1)
        mark("topk", 0)
        abi.dsv4_topk_select(params, o["scores"], q_index, o["idx"], stream=stream)
        mark("topk", 1)
    mark("attention", 0)
    if w.kind == "decode":
        abi.dsv4_sparse_mqa_attn(params, x["q"], x["win"], x["pool"], o["idx"], x["sink"], x["qpos"],
                                 x["q_index"], o["out"], ws, stream=stream)
    else:
        abi.dsv4_sparse_mqa_attn(params, x["q"], o["kv_rot"], o["pool"], o.get("idx") if w.kind != "hca" else None,
                                 x["sink"], x["pos"], None, o["out"], ws, stream=stream)
    mark("attention", 1)
