"""GPU-vs-oracle parity of the grouped output projection ("DeepSeek-V4" doc, Hybrid
attention (§2.3), grouped output projection: o_a_proj per head group, then o_b_proj),
through the C ABI dsv4_grouped_out_proj.

Tolerance, derived from the arithmetic (both products accumulate in fp32 on the tensor
cores; the intermediate u and the output y are stored in bf16, round to nearest even):
  |u - u_ref| <= 2^-9 |u_ref| + (K_a + 2) 2^-24 sum_c |wa_rc o_c|
  |y - y_ref| <= 2^-9 |y_ref| + sum_j |wb_kj| (2^-9 |u_ref_j| + acc_u_j) + (K_b + 2) 2^-24 sum_j |wb_kj u_j|
with u_ref, y_ref the fp64 oracle's values (u_ref from the oracle with an identity o_b_proj).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import dsv4_oracle as O

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
HALF_ULP = 2.0 ** -9


@pytest.fixture(scope="module")
def lib():
    from sparse_long_context_csa_b200 import abi, harness
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    return abi, harness


def _bounds(o, wa, wb):
    """Oracle u, y and the element-wise error bounds of the module docstring."""
    T, H, dv = o.shape
    g, dg, width = wa.shape
    u_ref = O.grouped_out_proj(o, wa, np.eye(g * dg))
    y_ref = O.grouped_out_proj(o, wa, wb)
    oa = np.abs(o.astype(np.float64)).reshape(T, g, width)
    mag_u = np.concatenate([oa[:, i] @ np.abs(wa[i].astype(np.float64)).T for i in range(g)], axis=1)
    acc_u = (width + 2) * U * mag_u
    tol_u = HALF_ULP * np.abs(u_ref) + acc_u
    awb = np.abs(wb.astype(np.float64))
    tol_y = HALF_ULP * np.abs(y_ref) + tol_u @ awb.T + (g * dg + 2) * U * (np.abs(u_ref) @ awb.T) * 1.01
    return u_ref, y_ref, tol_u, tol_y


def _run(lib, w, rows=None):
    abi, harness = lib
    host = synth.make_inputs(w)
    params = harness.params_for(w)
    x = harness.to_device(w, host)
    o = harness.make_outputs(w, params)
    harness.step(w, params, x, o)
    abi.dsv4_device_check()
    return host, o


def _check(host, o, rows):
    u_ref, y_ref, tol_u, tol_y = _bounds(host["o"][rows], host["wa"], host["wb"])
    gu = o["u"].float().cpu().numpy()[rows]
    gy = o["out"].float().cpu().numpy()[rows]
    bad_u = np.abs(gu - u_ref) > tol_u
    assert not bad_u.any(), f"u: {bad_u.sum()} elements out of bound, worst {np.abs(gu - u_ref).max():.3e}"
    bad_y = np.abs(gy - y_ref) > tol_y
    assert not bad_y.any(), f"y: {bad_y.sum()} elements out of bound, worst {np.abs(gy - y_ref).max():.3e}"
    return float(np.abs(gy - y_ref).max())


@pytest.mark.parametrize("T,g,dg,hidden", [(200, 8, 256, 512), (128, 1, 256, 256), (37, 4, 512, 768)])
def test_grouped_out_proj_small(lib, T, g, dg, hidden):
    """Ragged token counts (a partial 128-row tile), one group, and several tiles per group."""
    w = synth.WORKLOADS["out_proj_bf16"].replace(Sq=T, S=T, o_groups=g, o_rank=dg, hidden=hidden)
    host, o = _run(lib, w)
    _check(host, o, np.arange(T))


def test_grouped_out_proj_full_size_sampled_rows(lib):
    """The benchmarked size (8192 tokens, 64 heads x 512, 8 groups, o_lora_rank 1024,
    hidden 4096) on a strided sample of tokens plus the first and last ones."""
    w = synth.WORKLOADS["out_proj_bf16"]
    host, o = _run(lib, w)
    T = w.B * w.Sq
    rows = np.unique(np.concatenate([np.arange(8), np.linspace(0, T - 1, 40).astype(int), np.arange(T - 8, T)]))
    _check(host, o, rows)

