"""Host logic of bench.py that needs no GPU: the algorithmic work per part, the unit of each
workload, whether its steps are timed with L2 flushed, and the source hashes that tie each
recorded ncu DRAM figure to the kernel it was captured from."""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_sliding_window_attention_work_counts_window_keys_only():
    w = synth.WORKLOADS["swa_prefill_bf16"]
    qi, _ = synth.positions(w)
    keys = bench.attn_keys_per_query(w, qi)
    assert keys[0] == 1 and keys[127] == 128 and keys[-1] == 128
    work = bench.part_work(w, qi)
    assert set(work) == {"compress", "attention"}
    flops, nbytes = work["attention"]
    assert flops == float(keys.sum()) * 64 * (512 + 512) * 2
    # q + out + the rotated rows once; no index lists
    assert nbytes == 8192 * 64 * 1024 * 2 + 8192 * 512 * 2
    # RoPE only: rows read and the rotated rows written, no logits, no pool
    assert work["compress"] == (0.0, 2 * 8192 * 512 * 2)


def test_append_work_counts_closing_sequences():
    w = synth.WORKLOADS["csa_decode_append_bf16"]
    qi, _ = synth.positions(w)
    t = qi.reshape(-1)
    closing = int(((t + 1) % 4 == 0).sum())
    assert 0 < closing < 64
    work = bench.part_work(w, qi)
    assert set(work) == {"append"}
    per_seq = (4 * 512 * 2 + 8 + 512 * 2) + (4 * 128 * 2 + 8)
    per_entry = sum(2 * 8 * c * 2 + 8 * c * 4 + c * 2 for c in (512, 128))
    assert work["append"] == (0.0, 64 * per_seq + closing * per_entry)


def test_compress_work_counts_logits_only_when_pooling():
    dsa = synth.WORKLOADS["dsa_prefill_bf16"]   # m = 1: no compressor logits
    qi, _ = synth.positions(dsa)
    ch = 576 + 128
    assert bench.part_work(dsa, qi)["compress"][1] == 32768 * ch * 2 + 32768 * ch * 2 + 32768 * 576 * 2
    csa = synth.WORKLOADS["csa_prefill_bf16"]
    qi, _ = synth.positions(csa)
    ch = 512 + 128
    assert bench.part_work(csa, qi)["compress"][1] == 8192 * ch * 2 * 2 + 2048 * ch * 2 + 8192 * 512 * 2


def test_units_and_l2_policy_of_every_workload():
    units = {n: bench.per_step_kind(w) for n, w in synth.WORKLOADS.items()}
    assert units["csa_decode_bf16"] == units["csa_decode_append_bf16"] == "us/step"
    assert units["csa_prefill_bf16"] == units["swa_prefill_bf16"] == "tokens/s"
    flush = {n: bench.l2_flush_needed(w) for n, w in synth.WORKLOADS.items()}
    # inputs larger than L2 need no flush; the append's few rows and the tiny case do
    assert flush == {"tiny_csa_f32": True, "csa_prefill_bf16": False, "hca_prefill_bf16": False,
                     "csa_decode_bf16": False, "dsa_prefill_bf16": False, "swa_prefill_bf16": False,
                     "csa_decode_append_bf16": True, "out_proj_bf16": False}
    for n, w in synth.WORKLOADS.items():
        c = bench.config_of(w)
        assert c["workload"] == n and ("flushed" in c["l2"]) == flush[n]


def test_append_inputs_are_the_last_tokens_before_and_at_the_query():
    w = synth.WORKLOADS["csa_decode_append_bf16"]
    x = synth.make_inputs(w)
    assert x["kv"].shape == (8, 64, 512) and x["kI"].shape == (8, 64, 128)
    np.testing.assert_array_equal(x["t_hist"][-1], x["q_index"][:, 0])
    np.testing.assert_array_equal(np.diff(x["t_hist"], axis=0), 1)
    np.testing.assert_array_equal(x["pos_hist"], x["t_hist"])


def test_step_inputs_are_activations_that_exist():
    """The e2e leg copies these every step: they exist in the inputs (the logits only when
    m > 1), and no layer weight or decode-cache tensor is among them."""
    from sparse_long_context_csa_b200 import harness
    for name in ("tiny_csa_f32", "csa_decode_append_bf16"):
        w = synth.WORKLOADS[name]
        x = synth.make_inputs(w)
        assert all(k in x for k in harness.step_input_keys(w)), name  # nothing optional here (m > 1)
    for w in synth.WORKLOADS.values():
        keys = set(harness.step_input_keys(w))
        assert not keys & {"bias", "biasI", "sink", "pool", "poolI", "win"}


def _local_includes(name: str) -> set[str]:
    """The csrc headers a source file includes, followed through the headers themselves."""
    import re
    csrc = os.path.join(ROOT, "sparse_long_context_csa_b200", "csrc")
    seen, todo = set(), [name]
    while todo:
        text = open(os.path.join(csrc, todo.pop())).read()
        for inc in re.findall(r'^#include "([^"]+)"', text, flags=re.M):
            if inc not in seen and os.path.exists(os.path.join(csrc, inc)):
                seen.add(inc)
                todo.append(inc)
    return seen


def test_recorded_traffic_hashes_cover_each_kernel_and_its_headers():
    """A recorded ncu DRAM figure is tied to the SHA-256 of the kernel's source: its file up to
    the end marker, plus every csrc header the file includes.  The end marker must exist (else
    the figure would silently never apply), and no included header may be left out of the
    hash (else a change there would keep reporting the old figure)."""
    for (workload, part), (segments, sha, traffic) in bench.NCU_TRAFFIC.items():
        names = [n for n, _ in segments]
        main, end = segments[0]
        assert end is not None and end in open(os.path.join(
            ROOT, "sparse_long_context_csa_b200", "csrc", main)).read(), (workload, part, "end marker")
        missing = _local_includes(main) - set(names)
        assert not missing, f"{workload}/{part}: headers outside the hash: {sorted(missing)}"
        assert bench.kernel_source_sha(segments) is not None
        assert traffic > 0 and len(sha) == 64


def test_a_changed_kernel_reports_no_traffic(monkeypatch):
    rec = dict(bench.NCU_TRAFFIC)
    key = next(iter(rec))
    segments, sha, traffic = rec[key]
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, (segments, "0" * 64, traffic))
    assert bench.ncu_traffic(*key) is None
    monkeypatch.setitem(bench.NCU_TRAFFIC, key, (segments, bench.kernel_source_sha(segments), traffic))
    assert bench.ncu_traffic(*key) == traffic
