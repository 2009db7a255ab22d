"""dsv4_indexer_topk_noalloc: the indexer for callers that cannot allocate device memory.

Some hosts give a kernel library no allocator (they own every byte of device memory), and
some decode loops cannot call cudaMalloc / cudaFree because those calls may synchronise
the device.  The allocation-free entry point keeps its fp32 score rows in a fixed 16 MiB
array inside the library instead of a caller workspace.  This test calls it through the C
ABI twice in a row (the second call finds the first call's scores still in the array) and
requires the same index lists as the workspace entry point, which the parity tests pin to
the oracle; index lists are compared bit-exactly, as everywhere in the tests.  This file is
collected last so that a run stopping at its first failure has run every other test.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _setup(name, **over):
    from sparse_long_context_csa_b200 import abi, harness
    w = synth.WORKLOADS[name].replace(**over) if over else synth.WORKLOADS[name]
    sp = synth.cache_specs(w)
    specs = synth.tensor_specs(w)
    qi, _ = synth.positions(w)
    host = {"qI": synth.reshape(w, "qI", specs["qI"].full()), "wI": synth.reshape(w, "wI", specs["wI"].full()),
            "poolI": sp["poolI"].full().reshape(w.B, w.P_cap, w.cI), "q_index": qi}
    return abi, harness, w, harness.params_for(w), harness.to_device(w, host)


@pytest.mark.parametrize("name", ["tiny_csa_f32", "csa_prefill_bf16", "csa_decode_bf16"])
def test_noalloc_indexer_matches_workspace_entry_point(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi, harness, w, p, d = _setup(name)
    ws = torch.empty(max(abi.dsv4_workspace_bytes(p), 256), dtype=torch.uint8, device="cuda")
    ref = torch.full((w.B, w.Sq, w.topk), -7, dtype=torch.int32, device="cuda")
    abi.dsv4_indexer_topk(p, d["qI"], d["wI"], d["poolI"], d["q_index"], ref, ws)
    for call in range(2):
        got = torch.full((w.B, w.Sq, w.topk), -7, dtype=torch.int32, device="cuda")
        abi.dsv4_indexer_topk_noalloc(p, d["qI"], d["wI"], d["poolI"], d["q_index"], got)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}: index lists differ from the workspace entry point"
    assert int((ref >= 0).sum()) > 0

