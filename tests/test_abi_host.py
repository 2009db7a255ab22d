"""Host-side checks of libdsv4 that need no GPU: the library builds for sm_100a, loads,
exports every entry point include/dsv4.h declares, and rejects bad calls on the host
(those calls return before any CUDA call, so they are safe without a device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    from sparse_long_context_csa_b200 import abi, build
    build.build()
    abi.load()
    return abi


def _declared():
    src = open(os.path.join(ROOT, "include", "dsv4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsv4_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(abi):
    names = _declared()
    assert {"dsv4_compress_kv", "dsv4_indexer_topk", "dsv4_sparse_mqa_attn", "dsv4_csa_layer",
            "dsv4_hca_layer"} <= set(names)
    lib = ctypes.CDLL(abi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(abi.EXPORTED) == set(names)


def test_version_and_status_strings(abi):
    lib = abi.load()
    assert lib.dsv4_version() >= 100
    for code in range(8):
        assert lib.dsv4_status_string(code)
    assert b"unknown" in lib.dsv4_status_string(99)


def _params(abi, **kw):
    import synth
    from sparse_long_context_csa_b200 import harness
    return harness.params_for(synth.WORKLOADS["csa_prefill_bf16"], **kw)


FAKE = 0x10000  # 16-byte aligned fake device address: never dereferenced, validation fails first


def _attn(abi, p, **over):
    a = dict(q=FAKE, kv_win=FAKE, pool=FAKE, idx=FAKE, sink=FAKE, qpos=FAKE, q_index=None, out=FAKE)
    a.update(over)
    lib = abi.load()
    return lib.dsv4_sparse_mqa_attn(ctypes.byref(p) if p is not None else None, a["q"], a["kv_win"], a["pool"],
                                    a["idx"], a["sink"], a["qpos"], a["q_index"], a["out"], None, 0, None)


def test_attention_rejects_bad_arguments(abi):
    assert _attn(abi, None) == 1
    assert _attn(abi, _params(abi, dtype=7)) == 4
    assert _attn(abi, _params(abi, dv=500)) == 2                 # dv not a multiple of 32
    assert _attn(abi, _params(abi, dv=256)) == 2                 # rotate_out needs dv == D
    assert _attn(abi, _params(abi, R=63)) == 2                   # odd rope width
    assert _attn(abi, _params(abi, win_ring=64)) == 2            # ring shorter than the window
    assert _attn(abi, _params(abi), q=FAKE + 8) == 3             # misaligned
    assert _attn(abi, _params(abi), q=None) == 1
    assert _attn(abi, _params(abi), qpos=None) == 1              # rope_q needs positions
    assert _attn(abi, _params(abi, m=0)) == 2


def _attn_scores(abi, p, **over):
    a = dict(q=FAKE, kv_win=FAKE, pool=FAKE, scores=FAKE, sink=FAKE, qpos=FAKE, q_index=None, idx=FAKE, out=FAKE)
    a.update(over)
    lib = abi.load()
    return lib.dsv4_sparse_mqa_attn_scores(ctypes.byref(p) if p is not None else None, a["q"], a["kv_win"],
                                           a["pool"], a["scores"], a["sink"], a["qpos"], a["q_index"], a["idx"],
                                           a["out"], None, 0, None)


def test_attention_with_selection_rejects_bad_arguments(abi):
    """dsv4_sparse_mqa_attn_scores validates like dsv4_topk_select + dsv4_sparse_mqa_attn,
    on the host, before any launch (every call here fails validation)."""
    assert _attn_scores(abi, None) == 1
    assert _attn_scores(abi, _params(abi, dtype=7)) == 4
    assert _attn_scores(abi, _params(abi), scores=None) == 1     # the score rows are required
    assert _attn_scores(abi, _params(abi), idx=None) == 1        # ... and the lists' buffer
    assert _attn_scores(abi, _params(abi), pool=None) == 1       # lists need a pool
    assert _attn_scores(abi, _params(abi), scores=FAKE + 4) == 3
    assert _attn_scores(abi, _params(abi), idx=FAKE + 8) == 3
    assert _attn_scores(abi, _params(abi, topk=0)) == 2
    assert _attn_scores(abi, _params(abi, dv=256)) == 2          # rotate_out needs dv == D
    assert _attn_scores(abi, _params(abi), q=None) == 1
    assert _attn_scores(abi, _params(abi), qpos=None) == 1


def test_indexer_rejects_bad_arguments(abi):
    lib = abi.load()

    def call(p, ws=FAKE, ws_bytes=1 << 40, **over):
        a = dict(qI=FAKE, wI=FAKE, poolI=FAKE, q_index=None, idx=FAKE)
        a.update(over)
        return lib.dsv4_indexer_topk(ctypes.byref(p), a["qI"], a["wI"], a["poolI"], a["q_index"], a["idx"],
                                     ws, ws_bytes, None)

    assert call(_params(abi, nI=3)) == 2
    assert call(_params(abi, cI=96)) == 2
    assert call(_params(abi, topk=0)) == 2
    assert call(_params(abi), ws=None, ws_bytes=0) == 7
    assert call(_params(abi), ws_bytes=1024) == 7
    assert call(_params(abi), idx=None) == 1
    assert call(_params(abi), wI=FAKE + 4) == 3


def test_split_indexer_calls_reject_bad_arguments(abi):
    lib = abi.load()

    def scores(p, **over):
        a = dict(qI=FAKE, wI=FAKE, poolI=FAKE, q_index=None, scores=FAKE)
        a.update(over)
        return lib.dsv4_indexer_scores(ctypes.byref(p) if p is not None else None, a["qI"], a["wI"], a["poolI"],
                                       a["q_index"], a["scores"], None)

    def select(p, **over):
        a = dict(scores=FAKE, q_index=None, idx=FAKE)
        a.update(over)
        return lib.dsv4_topk_select(ctypes.byref(p) if p is not None else None, a["scores"], a["q_index"],
                                    a["idx"], None)

    assert scores(None) == 1
    assert scores(_params(abi, nI=3)) == 2
    assert scores(_params(abi, cI=96)) == 2
    assert scores(_params(abi), scores=None) == 1
    assert scores(_params(abi), scores=FAKE + 4) == 3
    assert scores(_params(abi, Sq=9000)) == 2          # more queries than tokens and no q_index
    assert scores(_params(abi, dtype=5)) == 4
    assert select(None) == 1
    assert select(_params(abi, topk=0)) == 2
    assert select(_params(abi, P_cap=0)) == 2
    assert select(_params(abi), idx=None) == 1
    assert select(_params(abi), scores=FAKE + 8) == 3
    assert select(_params(abi, Sq=9000)) == 2
    # empty batches return before any launch
    assert scores(_params(abi, B=0)) == 0
    assert select(_params(abi, B=0)) == 0


def test_decode_append_rejects_bad_arguments(abi):
    lib = abi.load()

    def call(p, c=512, apply_rope=1, **over):
        a = dict(x=FAKE, z=FAKE, bias=FAKE, pos=FAKE, t=FAKE, buf_x=FAKE, buf_z=FAKE, buf_pos=FAKE, win=FAKE,
                 pool=FAKE)
        a.update(over)
        return lib.dsv4_decode_append(ctypes.byref(p) if p is not None else None, c, a["x"], a["z"], a["bias"],
                                      a["pos"], a["t"], a["buf_x"], a["buf_z"], a["buf_pos"], apply_rope,
                                      a["win"], a["pool"], None)

    assert call(None) == 1
    assert call(_params(abi, win_ring=128), c=511) == 2                   # odd channel count
    assert call(_params(abi, win_ring=128), t=None) == 1
    assert call(_params(abi, win_ring=128), pos=None) == 1
    assert call(_params(abi, win_ring=128), buf_z=None) == 1              # logits given but nowhere to buffer them
    assert call(_params(abi, win_ring=0)) == 2              # a window ring of no rows
    assert call(_params(abi, win_ring=128, R=63)) == 2                    # odd rope width
    assert call(_params(abi, win_ring=128, R=130)) == 2                   # wider than the frequency table
    assert call(_params(abi, win_ring=128), apply_rope=2) == 1
    assert call(_params(abi, win_ring=128), buf_x=FAKE + 4) == 3
    assert call(_params(abi, win_ring=128, dtype=9)) == 4
    assert call(_params(abi, win_ring=128, B=0)) == 0                     # nothing to append: no launch


def test_compress_and_layers_reject_bad_arguments(abi):
    lib = abi.load()
    p = _params(abi)
    assert lib.dsv4_compress_kv(ctypes.byref(p), 511, FAKE, None, None, FAKE, 1, FAKE, None, None) == 2
    assert lib.dsv4_compress_kv(ctypes.byref(p), 512, FAKE, None, None, None, 1, FAKE, None, None) == 1
    assert lib.dsv4_compress_kv(ctypes.byref(p), 512, FAKE, None, None, FAKE, 0, FAKE, FAKE, None) == 1
    small = _params(abi, P_cap=100)  # S/m = 2048 entries do not fit
    assert lib.dsv4_compress_kv(ctypes.byref(small), 512, FAKE, None, None, FAKE, 1, FAKE, None, None) == 2
    # sliding-window layers: no pool (P_cap 0, pool NULL) -> only the rotated rows, which are required
    wide = _params(abi, R=130)  # RoPE frequencies are tabled for R <= 128
    assert lib.dsv4_compress_kv(ctypes.byref(wide), 512, FAKE, None, None, FAKE, 1, FAKE, None, None) == 2
    nopool = _params(abi, P_cap=0)
    assert lib.dsv4_compress_kv(ctypes.byref(nopool), 512, FAKE, None, None, FAKE, 1, None, None, None) == 1
    assert lib.dsv4_compress_kv(ctypes.byref(nopool), 512, FAKE, None, None, FAKE, 0, None, FAKE, None) == 1
    assert lib.dsv4_compress_kv(ctypes.byref(nopool), 512, FAKE, None, None, FAKE, 1, FAKE, FAKE, None) == 2
    assert lib.dsv4_compress_kv(ctypes.byref(p), 512, FAKE, None, None, FAKE, 1, None, FAKE, None) == 1
    assert lib.dsv4_compress_kv(ctypes.byref(nopool), 512, FAKE + 4, None, None, FAKE, 1, None, FAKE, None) == 3
    assert lib.dsv4_compress_kv(ctypes.byref(_params(abi, P_cap=0, B=0)), 512, FAKE, None, None, FAKE, 1, None,
                                FAKE, None) == 0
    args = [FAKE] * 17  # q .. idx, workspace
    assert lib.dsv4_csa_layer(ctypes.byref(_params(abi, Sq=1)), *args, 1 << 40, None) == 2   # prefill only
    assert lib.dsv4_csa_layer(ctypes.byref(p), *args, 16, None) == 7                          # workspace too small
    assert lib.dsv4_csa_layer(ctypes.byref(p), *args[:16], None, 1 << 40, None) == 7
    assert lib.dsv4_hca_layer(ctypes.byref(p), *([FAKE] * 10), 0, None) == 2              # overlap=1 is CSA


def test_workspace_is_a_pure_function_of_params(abi):
    import synth
    from sparse_long_context_csa_b200 import harness
    sizes = {n: abi.dsv4_workspace_bytes(harness.params_for(w)) for n, w in synth.WORKLOADS.items()}
    assert sizes["hca_prefill_bf16"] == 0                      # no indexer
    assert sizes["csa_prefill_bf16"] == 8192 * 512 * 4 + 8192 * 2048 * 4
    # decode keeps no layer idx; its attention partials (5 key splits x 64 queries) dominate
    # 64 queries of 128 window + 2048 selected keys: two key splits per query
    assert sizes["csa_decode_bf16"] == max(64 * 32768 * 4, 64 * 2 * 64 * (512 + 2) * 4)
    assert sizes["dsa_prefill_bf16"] == 32768 * 2048 * 4 + (256 << 20)
    assert abi.dsv4_workspace_bytes(harness.params_for(synth.WORKLOADS["tiny_csa_f32"])) == \
        abi.dsv4_workspace_bytes(harness.params_for(synth.WORKLOADS["tiny_csa_f32"]))


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No CPU fallback: without the built library the binding raises instead of computing."""
    from sparse_long_context_csa_b200 import abi as mod
    monkeypatch.setattr(mod, "_lib", None)
    with pytest.raises(ImportError):
        mod.load(str(tmp_path / "libdsv4.so"))


def test_product_package_never_imports_the_oracle():
    """The CPU oracle is test infrastructure: nothing in the package refers to it."""
    pkg = os.path.join(ROOT, "sparse_long_context_csa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, flags=re.M), f
                assert "dsv4_oracle" not in src, f


def test_noalloc_indexer_rejects_pools_beyond_its_scratch(abi):
    """A pool of more entries than the fixed score scratch holds (4,194,304 fp32 scores) is
    refused with DSV4_ERR_SHAPE on the host, before the scratch is looked up or any kernel is
    enqueued: the fake addresses below are never dereferenced."""
    lib = abi.load()
    p = _params(abi, B=64, S=131072, Sq=1, P_cap=(4 << 20) + 1, topk=2048)
    st = lib.dsv4_indexer_topk_noalloc(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None)
    assert st == 2
    # at the limit the size check passes and the call goes on to the device (not made here)


def test_grouped_out_proj_rejects_untiled_sizes_on_the_host(abi):
    """Sizes the tensor-core tiles do not cover, float32 activations, null or misaligned
    pointers are refused before any CUDA call (fake addresses, never dereferenced)."""
    import synth
    from sparse_long_context_csa_b200 import harness
    lib = abi.load()
    w = synth.WORKLOADS["out_proj_bf16"]
    p = harness.params_for(w)
    ok = dict(T=16, groups=8, dg=256, hidden=512)
    cases = [(dict(dg=200), 2), (dict(hidden=300), 2), (dict(groups=3), 2), (dict(T=-1), 2)]
    for bad, want in cases:
        kw = {**ok, **bad}
        st = lib.dsv4_grouped_out_proj(ctypes.byref(p), kw["T"], kw["groups"], kw["dg"], kw["hidden"],
                                       FAKE, FAKE, FAKE, FAKE, FAKE, None)
        assert st == want, (bad, st)
    st = lib.dsv4_grouped_out_proj(ctypes.byref(p), 16, 8, 256, 512, FAKE, FAKE, None, FAKE, FAKE, None)
    assert st == 1
    st = lib.dsv4_grouped_out_proj(ctypes.byref(p), 16, 8, 256, 512, FAKE + 8, FAKE, FAKE, FAKE, FAKE, None)
    assert st == 3
    p32 = harness.params_for(w.replace(dtype="f32"))
    st = lib.dsv4_grouped_out_proj(ctypes.byref(p32), 16, 8, 256, 512, FAKE, FAKE, FAKE, FAKE, FAKE, None)
    assert st == 2
