"""ctypes binding of libdsv4 (include/dsv4.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch tensors
(or None for optional NULL pointers) that already live on the GPU, passes their
device pointers, and raises ``Dsv4Error`` when the library returns a non-zero status.
No arithmetic of the method happens in Python.  The library must have been built
(``python -m sparse_long_context_csa_b200.build``); loading fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsv4.so")

F32, BF16 = 0, 1
STATUS = {0: "DSV4_OK", 1: "DSV4_ERR_ARG", 2: "DSV4_ERR_SHAPE", 3: "DSV4_ERR_ALIGN", 4: "DSV4_ERR_DTYPE",
          5: "DSV4_ERR_CUDA", 6: "DSV4_ERR_DEVICE_CHECK", 7: "DSV4_ERR_WORKSPACE"}

EXPORTED = ("dsv4_compress_kv", "dsv4_indexer_topk", "dsv4_sparse_mqa_attn", "dsv4_csa_layer",
            "dsv4_hca_layer", "dsv4_workspace_bytes", "dsv4_status_string", "dsv4_version",
            "dsv4_launch_count", "dsv4_indexer_topk_noalloc", "dsv4_device_check", "dsv4_indexer_scores",
            "dsv4_topk_select", "dsv4_decode_append", "dsv4_grouped_out_proj", "dsv4_set_index_checks",
            "dsv4_index_checks", "dsv4_sparse_mqa_attn_scores")


class Dsv4Error(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({msg})")
        self.status = status


class Dsv4Params(ctypes.Structure):
    """Mirror of ``dsv4_params`` (field order and types must match include/dsv4.h)."""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "S", "Sq", "H", "D", "R", "dv", "n_win", "win_ring", "m", "overlap", "P_cap",
                 "nI", "cI", "topk")] + \
               [("scale", ctypes.c_float), ("rope_theta", ctypes.c_float)] + \
               [(n, ctypes.c_int32) for n in ("rope_q", "rotate_out", "dtype")]

    def __repr__(self):
        return "Dsv4Params(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdsv4.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m sparse_long_context_csa_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Dsv4Params)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.dsv4_compress_kv.argtypes = [P, i32, vp, vp, vp, vp, i32, vp, vp, vp]
    lib.dsv4_indexer_topk.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsv4_indexer_topk_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.dsv4_indexer_scores.argtypes = [P, vp, vp, vp, vp, vp, vp]
    lib.dsv4_topk_select.argtypes = [P, vp, vp, vp, vp]
    lib.dsv4_decode_append.argtypes = [P, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp]
    lib.dsv4_sparse_mqa_attn.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsv4_sparse_mqa_attn_scores.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsv4_csa_layer.argtypes = [P] + [vp] * 17 + [sz, vp]
    lib.dsv4_hca_layer.argtypes = [P] + [vp] * 10 + [sz, vp]
    lib.dsv4_grouped_out_proj.argtypes = [P, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.dsv4_set_index_checks.argtypes = [i32]
    lib.dsv4_set_index_checks.restype = None
    lib.dsv4_index_checks.restype = i32
    lib.dsv4_workspace_bytes.argtypes = [P]
    lib.dsv4_workspace_bytes.restype = sz
    lib.dsv4_status_string.argtypes = [ctypes.c_int]
    lib.dsv4_status_string.restype = ctypes.c_char_p
    lib.dsv4_version.restype = i32
    lib.dsv4_launch_count.restype = ctypes.c_uint64
    lib.dsv4_device_check.argtypes = [vp]
    lib.dsv4_device_check.restype = ctypes.c_int
    for fn in ("dsv4_compress_kv", "dsv4_indexer_topk", "dsv4_sparse_mqa_attn", "dsv4_csa_layer",
               "dsv4_hca_layer", "dsv4_indexer_topk_noalloc", "dsv4_indexer_scores", "dsv4_topk_select",
               "dsv4_decode_append", "dsv4_grouped_out_proj", "dsv4_sparse_mqa_attn_scores"):
        getattr(lib, fn).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise Dsv4Error(fn, st, load().dsv4_status_string(st).decode())


def dsv4_device_check(stream=None) -> None:
    """Synchronise the stream and raise if a kernel reported a device-side failure."""
    _check("dsv4_device_check", load().dsv4_device_check(_stream(stream)))


def dsv4_launch_count() -> int:
    return int(load().dsv4_launch_count())


def dsv4_workspace_bytes(params: Dsv4Params) -> int:
    return int(load().dsv4_workspace_bytes(ctypes.byref(params)))


def dsv4_compress_kv(params, c, x, z, bias, pos, apply_rope, pool, x_rot, stream=None):
    _check("dsv4_compress_kv", load().dsv4_compress_kv(
        ctypes.byref(params), int(c), _ptr(x), _ptr(z), _ptr(bias), _ptr(pos), int(apply_rope), _ptr(pool),
        _ptr(x_rot), _stream(stream)))


def dsv4_indexer_topk(params, qI, wI, poolI, q_index, idx, workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None \
        else (ws_bytes or 0)
    _check("dsv4_indexer_topk", load().dsv4_indexer_topk(
        ctypes.byref(params), _ptr(qI), _ptr(wI), _ptr(poolI), _ptr(q_index), _ptr(idx), _ptr(workspace),
        ws_bytes, _stream(stream)))


def dsv4_indexer_topk_noalloc(params, qI, wI, poolI, q_index, idx, stream=None):
    """dsv4_indexer_topk without a workspace: scores go to the library's fixed device scratch."""
    _check("dsv4_indexer_topk_noalloc", load().dsv4_indexer_topk_noalloc(
        ctypes.byref(params), _ptr(qI), _ptr(wI), _ptr(poolI), _ptr(q_index), _ptr(idx), _stream(stream)))


def dsv4_indexer_scores(params, qI, wI, poolI, q_index, scores, stream=None):
    """Lightning Indexer scores only: scores[B*Sq, P_cap] f32 (entries past each row's visible count untouched)."""
    _check("dsv4_indexer_scores", load().dsv4_indexer_scores(
        ctypes.byref(params), _ptr(qI), _ptr(wI), _ptr(poolI), _ptr(q_index), _ptr(scores), _stream(stream)))


def dsv4_topk_select(params, scores, q_index, idx, stream=None):
    """Per-query top-k over given score rows: idx[B,Sq,topk] ascending entries, then -1."""
    _check("dsv4_topk_select", load().dsv4_topk_select(
        ctypes.byref(params), _ptr(scores), _ptr(q_index), _ptr(idx), _stream(stream)))


def dsv4_decode_append(params, c, x, z, bias, pos, t, buf_x, buf_z, buf_pos, apply_rope, win, pool, stream=None):
    """Append one token per sequence to the decode cache (buffer, window ring, pool)."""
    _check("dsv4_decode_append", load().dsv4_decode_append(
        ctypes.byref(params), c, _ptr(x), _ptr(z), _ptr(bias), _ptr(pos), _ptr(t), _ptr(buf_x), _ptr(buf_z),
        _ptr(buf_pos), apply_rope, _ptr(win), _ptr(pool), _stream(stream)))


def dsv4_sparse_mqa_attn(params, q, kv_win, pool, idx, sink, qpos, q_index, out, workspace=None,
                         ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None \
        else (ws_bytes or 0)
    _check("dsv4_sparse_mqa_attn", load().dsv4_sparse_mqa_attn(
        ctypes.byref(params), _ptr(q), _ptr(kv_win), _ptr(pool), _ptr(idx), _ptr(sink), _ptr(qpos),
        _ptr(q_index), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


def dsv4_sparse_mqa_attn_scores(params, q, kv_win, pool, scores, sink, qpos, q_index, idx, out, workspace=None,
                                ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None \
        else (ws_bytes or 0)
    _check("dsv4_sparse_mqa_attn_scores", load().dsv4_sparse_mqa_attn_scores(
        ctypes.byref(params), _ptr(q), _ptr(kv_win), _ptr(pool), _ptr(scores), _ptr(sink), _ptr(qpos),
        _ptr(q_index), _ptr(idx), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


def dsv4_csa_layer(params, q, kv, z, bias, qI, wI, kI, zI, biasI, sink, pos, out, pool, poolI, kv_rot, idx,
                   workspace, ws_bytes=None, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None \
        else (ws_bytes or 0)
    _check("dsv4_csa_layer", load().dsv4_csa_layer(
        ctypes.byref(params), _ptr(q), _ptr(kv), _ptr(z), _ptr(bias), _ptr(qI), _ptr(wI), _ptr(kI), _ptr(zI),
        _ptr(biasI), _ptr(sink), _ptr(pos), _ptr(out), _ptr(pool), _ptr(poolI), _ptr(kv_rot), _ptr(idx),
        _ptr(workspace), ws_bytes, _stream(stream)))


def dsv4_hca_layer(params, q, kv, z, bias, sink, pos, out, pool, kv_rot, workspace=None, ws_bytes=None,
                   stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if ws_bytes is None and workspace is not None \
        else (ws_bytes or 0)
    _check("dsv4_hca_layer", load().dsv4_hca_layer(
        ctypes.byref(params), _ptr(q), _ptr(kv), _ptr(z), _ptr(bias), _ptr(sink), _ptr(pos), _ptr(out),
        _ptr(pool), _ptr(kv_rot), _ptr(workspace), ws_bytes, _stream(stream)))


def dsv4_grouped_out_proj(params, T, groups, dg, hidden, o, wa, wb, u, y, stream=None):
    _check("dsv4_grouped_out_proj",
           load().dsv4_grouped_out_proj(ctypes.byref(params), T, groups, dg, hidden, _ptr(o), _ptr(wa), _ptr(wb),
                                        _ptr(u), _ptr(y), _stream(stream)))


def dsv4_set_index_checks(on: bool) -> None:
    load().dsv4_set_index_checks(1 if on else 0)


def dsv4_index_checks() -> bool:
    return bool(load().dsv4_index_checks())
