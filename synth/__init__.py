"""Seeded synthetic inputs shaped like the five workloads of the attention core.

This module draws random numbers and casts them to the storage dtype; it holds
none of the method's arithmetic.  The CPU oracle and the CUDA path both take
their inputs from here, so it is the only module they share.

Every tensor is drawn in blocks of ``CHUNK`` leading rows; block ``k`` of tensor
``stream`` comes from ``numpy.random.default_rng([seed, stream, k])``, so any
subset of rows can be regenerated without drawing the rest (the oracle uses this
to check sampled rows of the largest workloads).

Distributions (per tensor, over its last dimension ``d``):
  q, kv, qI, kI, decode pool / indexer pool / window rows: N(0,1)/sqrt(d)
  compressor logits z, zI: N(0,1);  per-slot compressor bias: 0.1 N(0,1)
  indexer head weights wI: N(0,1)/sqrt(n_I);  sink logits: N(0,1)
bf16 workloads round every value to the nearest bf16 (ties to even) here, so
both sides read identical values.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 256
BASE_SEED = 20261202

STREAMS = {
    "q": 1, "kv": 2, "z": 3, "bias": 4, "qI": 5, "wI": 6, "kI": 7, "zI": 8,
    "biasI": 9, "sink": 10, "pool": 11, "poolI": 12, "win": 13, "q_index": 14,
    "o": 16, "wa": 17, "wb": 18,
}
# (stream 15 draws the offsets of strided_selection)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    config_id: int
    kind: str            # "csa" | "hca" | "decode" | "dsa" | "swa" (window only) | "append" | "outproj"
    dtype: str           # "f32" | "bf16"
    B: int
    S: int               # tokens in the sequence (prefill) / cache length (decode)
    Sq: int              # query tokens per sequence
    H: int
    D: int
    R: int
    dv: int
    n_win: int
    m: int
    overlap: int
    nI: int
    cI: int
    topk: int
    theta: float
    rotate_out: int
    P_cap: int           # pool capacity (entries per sequence)
    win_ring: int = 0    # >0: window rows live in a ring of this many slots
    qindex_spread: int = 0
    o_groups: int = 0    # grouped output projection: head groups, o_lora_rank, hidden_size
    o_rank: int = 0
    hidden: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def seed(self) -> int:
        return BASE_SEED + self.config_id

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_csa_f32": Workload("tiny_csa_f32", 0, "csa", "f32", B=1, S=512, Sq=512, H=8, D=128,
                             R=64, dv=128, n_win=64, m=4, overlap=1, nI=4, cI=64, topk=32,
                             theta=160000.0, rotate_out=1, P_cap=128),
    "csa_prefill_bf16": Workload("csa_prefill_bf16", 1, "csa", "bf16", B=1, S=8192, Sq=8192,
                                 H=64, D=512, R=64, dv=512, n_win=128, m=4, overlap=1, nI=8,
                                 cI=128, topk=512, theta=160000.0, rotate_out=1, P_cap=2048),
    "hca_prefill_bf16": Workload("hca_prefill_bf16", 2, "hca", "bf16", B=1, S=65536, Sq=65536,
                                 H=64, D=512, R=64, dv=512, n_win=128, m=128, overlap=0, nI=0,
                                 cI=0, topk=0, theta=160000.0, rotate_out=1, P_cap=512),
    "csa_decode_bf16": Workload("csa_decode_bf16", 3, "decode", "bf16", B=64, S=131072, Sq=1,
                                H=64, D=512, R=64, dv=512, n_win=128, m=4, overlap=1, nI=8,
                                cI=128, topk=2048, theta=160000.0, rotate_out=1, P_cap=32768,
                                win_ring=128, qindex_spread=1024),
    "dsa_prefill_bf16": Workload("dsa_prefill_bf16", 4, "dsa", "bf16", B=1, S=32768, Sq=32768,
                                 H=64, D=576, R=64, dv=512, n_win=0, m=1, overlap=0, nI=1,
                                 cI=128, topk=2048, theta=10000.0, rotate_out=0, P_cap=32768),
    # a sliding_attention layer of the same shape as the CSA prefill: RoPE of the K=V rows,
    # then attention over the 128-token window alone (no pool, no indexer)
    "swa_prefill_bf16": Workload("swa_prefill_bf16", 5, "swa", "bf16", B=1, S=8192, Sq=8192,
                                 H=64, D=512, R=64, dv=512, n_win=128, m=1, overlap=0, nI=0,
                                 cI=0, topk=0, theta=10000.0, rotate_out=1, P_cap=0),
    # one decode-cache append per sequence of the CSA decode cache: the K=V stream (buffer,
    # window ring, pool) and the indexer-key stream (buffer, pool)
    "csa_decode_append_bf16": Workload("csa_decode_append_bf16", 6, "append", "bf16", B=64, S=131072,
                                       Sq=1, H=64, D=512, R=64, dv=512, n_win=128, m=4, overlap=1,
                                       nI=8, cI=128, topk=2048, theta=160000.0, rotate_out=1,
                                       P_cap=32768, win_ring=128, qindex_spread=1024),
    # the grouped output projection of the CSA prefill's attention output (8192 tokens, 64
    # heads x 512): o_groups 8, o_lora_rank 1024, hidden_size 4096 (DeepseekV4Config defaults)
    "out_proj_bf16": Workload("out_proj_bf16", 7, "outproj", "bf16", B=1, S=8192, Sq=8192, H=64, D=512,
                              R=0, dv=512, n_win=0, m=1, overlap=0, nI=0, cI=0, topk=0, theta=10000.0,
                              rotate_out=0, P_cap=0, o_groups=8, o_rank=1024, hidden=4096),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (r.astype(np.uint32) << 16).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class TensorSpec:
    """A seeded N(0,1)*scale tensor whose leading dimension is drawn in chunks."""
    seed: int
    stream: int
    shape: tuple
    scale: float
    bf16: bool

    @property
    def nrows(self) -> int:
        return self.shape[0]

    @property
    def row_shape(self) -> tuple:
        return tuple(self.shape[1:])

    def chunk(self, k: int) -> np.ndarray:
        lo = k * CHUNK
        n = min(CHUNK, self.nrows - lo)
        rng = np.random.default_rng([self.seed, self.stream, k])
        a = rng.standard_normal((n,) + self.row_shape, dtype=np.float32)
        a *= np.float32(self.scale)
        return round_to_bf16(a) if self.bf16 else a

    def rows(self, lo: int, hi: int) -> np.ndarray:
        out = np.empty((hi - lo,) + self.row_shape, dtype=np.float32)
        for k in range(lo // CHUNK, (hi - 1) // CHUNK + 1 if hi > lo else 0):
            c = self.chunk(k)
            a, b = max(lo, k * CHUNK), min(hi, k * CHUNK + c.shape[0])
            out[a - lo:b - lo] = c[a - k * CHUNK:b - k * CHUNK]
        return out

    def take(self, row_ids) -> np.ndarray:
        row_ids = list(row_ids)
        out = np.empty((len(row_ids),) + self.row_shape, dtype=np.float32)
        by_chunk = {}
        for i, r in enumerate(row_ids):
            by_chunk.setdefault(r // CHUNK, []).append((i, r))
        for k, lst in by_chunk.items():
            c = self.chunk(k)
            for i, r in lst:
                out[i] = c[r - k * CHUNK]
        return out

    def full(self, threads: int = 8) -> np.ndarray:
        out = np.empty(self.shape, dtype=np.float32)
        nchunks = (self.nrows + CHUNK - 1) // CHUNK

        def fill(k):
            c = self.chunk(k)
            out[k * CHUNK:k * CHUNK + c.shape[0]] = c

        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(fill, range(nchunks)))
        return out


def tensor_specs(w: Workload, gains: dict | None = None) -> dict:
    """Specs of every input tensor of workload ``w`` (leading dims flattened)."""
    gains = gains or {}
    bf = w.dtype == "bf16"
    s = w.seed

    def spec(name, shape, scale, bf16=bf):
        return TensorSpec(s, STREAMS[name], tuple(shape), float(scale) * gains.get(name, 1.0), bf16)

    if w.kind == "append":
        # rows of the last Lw tokens of every sequence, token-major ([Lw, B, c]); the last
        # one is the token the step appends
        lw = 2 * w.m if w.overlap else w.m
        return {"kv": spec("kv", (lw * w.B, w.D), 1 / math.sqrt(w.D)),
                "z": spec("z", (lw * w.B, w.D), 1.0),
                "bias": spec("bias", (lw, w.D), 0.1, bf16=False),
                "kI": spec("kI", (lw * w.B, w.cI), 1 / math.sqrt(w.cI)),
                "zI": spec("zI", (lw * w.B, w.cI), 1.0),
                "biasI": spec("biasI", (lw, w.cI), 0.1, bf16=False)}
    if w.kind == "outproj":
        # attention outputs (one value row's scale) and the two projection weights, each
        # N(0,1)/sqrt(fan_in)
        width = (w.H // w.o_groups) * w.dv
        return {"o": spec("o", (w.B * w.Sq, w.H, w.dv), 1 / math.sqrt(w.dv)),
                "wa": spec("wa", (w.o_groups * w.o_rank, width), 1 / math.sqrt(width)),
                "wb": spec("wb", (w.hidden, w.o_groups * w.o_rank), 1 / math.sqrt(w.o_groups * w.o_rank))}
    specs = {
        "q": spec("q", (w.B * w.Sq, w.H, w.D), 1 / math.sqrt(w.D)),
        "sink": spec("sink", (w.H,), 1.0, bf16=False),
    }
    if w.kind == "decode":
        specs["pool"] = spec("pool", (w.B * w.P_cap, w.D), 1 / math.sqrt(w.D))
        specs["poolI"] = spec("poolI", (w.B * w.P_cap, w.cI), 1 / math.sqrt(w.cI))
        specs["win"] = spec("win", (w.B * w.win_ring, w.D), 1 / math.sqrt(w.D))
    else:
        lw = (2 * w.m if w.overlap else w.m)
        specs["kv"] = spec("kv", (w.B * w.S, w.D), 1 / math.sqrt(w.D))
        if w.m > 1:
            specs["z"] = spec("z", (w.B * w.S, w.D), 1.0)
            specs["bias"] = spec("bias", (lw, w.D), 0.1, bf16=False)
    if w.nI > 0:
        specs["qI"] = spec("qI", (w.B * w.Sq, w.nI, w.cI), 1 / math.sqrt(w.cI))
        specs["wI"] = spec("wI", (w.B * w.Sq, w.nI), 1 / math.sqrt(w.nI), bf16=False)
        if w.kind != "decode":
            specs["kI"] = spec("kI", (w.B * w.S, w.cI), 1 / math.sqrt(w.cI))
            if w.m > 1:
                lw = (2 * w.m if w.overlap else w.m)
                specs["zI"] = spec("zI", (w.B * w.S, w.cI), 1.0)
                specs["biasI"] = spec("biasI", (lw, w.cI), 0.1, bf16=False)
    return specs


def positions(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    """(q_index [B,Sq] int64 cache indices, qpos [B,Sq] int64 RoPE positions).

    Prefill: query s sits at cache index s.  Decode: each sequence's new token
    sits at S-1-U{0..qindex_spread-1}, drawn from stream ``q_index``.
    """
    if w.kind in ("decode", "append"):
        rng = np.random.default_rng([w.seed, STREAMS["q_index"], 0])
        qi = (w.S - 1 - rng.integers(0, w.qindex_spread, size=(w.B, 1))).astype(np.int64)
    else:
        qi = np.tile(np.arange(w.Sq, dtype=np.int64), (w.B, 1))
    return qi, qi.copy()


def token_positions(w: Workload) -> np.ndarray:
    """RoPE positions of the cached tokens [B,S] (prefill: 0..S-1)."""
    return np.tile(np.arange(w.S, dtype=np.int64), (w.B, 1))


def reshape(w: Workload, name: str, a: np.ndarray) -> np.ndarray:
    """Unflatten a full tensor drawn from ``tensor_specs`` to its logical shape."""
    if w.kind == "append":
        return a.reshape((-1, w.B) + a.shape[1:]) if name in ("kv", "z", "kI", "zI") else a
    shapes = {
        "q": (w.B, w.Sq, w.H, w.D), "kv": (w.B, w.S, w.D), "z": (w.B, w.S, w.D),
        "qI": (w.B, w.Sq, w.nI, w.cI), "wI": (w.B, w.Sq, w.nI), "kI": (w.B, w.S, w.cI),
        "zI": (w.B, w.S, w.cI), "pool": (w.B, w.P_cap, w.D), "poolI": (w.B, w.P_cap, w.cI),
        "win": (w.B, w.win_ring, w.D), "o": (w.B * w.Sq, w.H, w.dv),
        "wa": (w.o_groups, w.o_rank, (w.H // w.o_groups) * w.dv if w.o_groups else 0),
    }
    return a.reshape(shapes[name]) if name in shapes else a


def make_inputs(w: Workload, gains: dict | None = None, threads: int = 8) -> dict:
    """All inputs of ``w`` as float32 numpy arrays in their logical shapes, plus positions."""
    out = {name: reshape(w, name, sp.full(threads)) for name, sp in tensor_specs(w, gains).items()}
    out["q_index"], out["qpos"] = positions(w)
    if w.kind == "append":
        # cache index (= position) of history token k of sequence b: q_index[b] - (Lw-1-k)
        lw = out["kv"].shape[0]
        t = out["q_index"][:, 0][None, :] - np.arange(lw - 1, -1, -1, dtype=np.int64)[:, None]
        out["t_hist"] = t.astype(np.int32)
        out["pos_hist"] = t.astype(np.int64)
    elif w.kind not in ("decode", "outproj"):
        out["pos"] = token_positions(w)
    return out


def strided_selection(w: Workload, q_index: np.ndarray, stream: int = 15) -> np.ndarray:
    """A valid index list per query for attention-only tests: [B,Sq,topk] int32.

    Query (b,s) at cache index t keeps n = min(topk, vis) of its vis visible entries,
    entry k = floor((k + u) * vis / n) for a seeded offset u in [0,1): distinct,
    ascending, spread over the whole visible range; the remaining slots are -1.
    """
    rng = np.random.default_rng([w.seed, stream, 0])
    t = q_index.reshape(-1).astype(np.int64)
    vis = np.minimum((t + 1) // w.m, w.P_cap)
    n = np.minimum(vis, w.topk)
    u = rng.random(t.shape[0])
    k = np.arange(w.topk, dtype=np.float64)[None, :]
    nn = np.maximum(n, 1)[:, None].astype(np.float64)
    sel = np.floor((k + u[:, None]) * vis[:, None] / nn).astype(np.int64)
    sel = np.where(k < n[:, None], sel, -1)
    return sel.reshape(w.B, w.Sq, w.topk).astype(np.int32)


def cache_specs(w: Workload, gains: dict | None = None) -> dict:
    """Specs of a pre-filled cache for kernel-level tests of any workload:
    pool [B*P_cap, D], poolI [B*P_cap, cI] and window rows [B*(win_ring or S), D]."""
    gains = gains or {}
    bf = w.dtype == "bf16"

    def spec(name, shape, scale):
        return TensorSpec(w.seed, STREAMS[name], tuple(shape), float(scale) * gains.get(name, 1.0), bf)

    rows = w.win_ring if w.win_ring else w.S
    out = {"pool": spec("pool", (w.B * w.P_cap, w.D), 1 / math.sqrt(w.D)),
           "win": spec("win", (w.B * rows, w.D), 1 / math.sqrt(w.D))}
    if w.nI > 0:
        out["poolI"] = spec("poolI", (w.B * w.P_cap, w.cI), 1 / math.sqrt(w.cI))
    return out
