"""Pins of the fp64 oracle against facts the pages and mathematics fix.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one window) fails it.
None of these tests re-types an oracle formula: each compares the oracle with
the pages' worked example, a closed form, an invariance, a textbook routine or
brute force.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import expit, logsumexp

from oracle import dsv4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden_sections(name):
    sec, out = None, {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                sec = line.strip("[]")
                out[sec] = []
            else:
                out[sec].append(line)
    return out


# ---------------------------------------------------------------- mask example
def test_mask_example_grid():
    g = _read_golden_sections("mask_example_16tok.txt")
    S, win, m_csa, m_hca, k = 16, 8, 4, 8, 2
    for t in range(S):
        row = ["0"] * S
        for j in O.window_tokens(t, win):
            row[j] = "1"
        assert "".join(row) == g["sliding"][t], t
        vis = O.visible_entries(t, m_hca)
        hca = "".join("1" if w < vis else "0" for w in range(S // m_hca))
        assert hca == g["hca_entries"][t], t
        vis_c = O.visible_entries(t, m_csa)
        scores = np.random.default_rng(t).standard_normal(vis_c)
        _, padded = O.topk_select_row(scores, k)
        assert int((padded >= 0).sum()) == int(g["csa_filled_slots"][t]), t
        assert all(p == -1 for p in padded[(padded >= 0).sum():])


# ---------------------------------------------------------------- RoPE
def _rope_complex(x, pos, R, theta, sign=1.0):
    """Independent restatement: each channel pair is a complex number times e^{i angle}."""
    x = np.asarray(x, dtype=np.float64)
    c = x.shape[-1]
    zc = x[..., c - R::2] + 1j * x[..., c - R + 1::2]
    freqs = np.array([theta ** (-(2.0 * k) / R) for k in range(R // 2)])
    zc = zc * np.exp(1j * sign * np.asarray(pos, dtype=np.float64)[..., None] * freqs)
    out = x.copy()
    out[..., c - R::2] = zc.real
    out[..., c - R + 1::2] = zc.imag
    return out


def test_rope_closed_form_and_algebra():
    rng = np.random.default_rng(0)
    R, theta = 8, 10000.0
    # unit vector on pair k at position 1 lands at (cos f_k, sin f_k), f_k = theta^(-2k/R)
    for k in range(R // 2):
        e = np.zeros(12)
        e[12 - R + 2 * k] = 1.0
        r = O.rope_rotate(e, 1, R, theta)
        f = theta ** (-2.0 * k / R)
        assert r[12 - R + 2 * k] == pytest.approx(math.cos(f), abs=1e-15)
        assert r[12 - R + 2 * k + 1] == pytest.approx(math.sin(f), abs=1e-15)
        assert np.all(r[: 12 - R] == 0)
    x = rng.standard_normal((5, 16))
    pos = np.array([0, 3, 77, 1000, 131071])
    r = O.rope_rotate(x, pos, R, theta)
    np.testing.assert_allclose(r, _rope_complex(x, pos, R, theta), atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_array_equal(r[:, : 16 - R], x[:, : 16 - R])
    back = O.rope_rotate(r, pos, R, theta, sign=-1.0)
    np.testing.assert_allclose(back, x, atol=1e-12)
    # relative-position property: <R(p)a, R(p')b> depends only on p - p'
    a, b = rng.standard_normal(16), rng.standard_normal(16)
    d1 = O.rope_rotate(a, 10, R, theta) @ O.rope_rotate(b, 4, R, theta)
    d2 = O.rope_rotate(a, 1006, R, theta) @ O.rope_rotate(b, 1000, R, theta)
    assert d1 == pytest.approx(d2, abs=1e-11)


# ---------------------------------------------------------------- compressor
def _expected_mean(x, w, m, overlap):
    S = x.shape[0]
    lo = max(0, (w - 1) * m) if overlap else w * m
    hi = min(S, (w + 1) * m)
    return x[lo:hi].mean(axis=0)


@pytest.mark.parametrize("overlap", [0, 1])
def test_compress_zero_logits_is_window_mean(overlap):
    rng = np.random.default_rng(1)
    B, S, c, m = 2, 40, 6, 4
    x = rng.standard_normal((B, S, c))
    pool = O.compress(x, np.zeros((B, S, c)), np.zeros((2 * m if overlap else m, c)), None,
                      m=m, overlap=overlap, apply_rope=False)
    assert pool.shape == (B, S // m, c)
    for b in range(B):
        for w in range(S // m):
            np.testing.assert_allclose(pool[b, w], _expected_mean(x[b], w, m, overlap), atol=1e-14)
    # no logits and no bias at all is the same mean
    pool2 = O.compress(x, None, None, None, m=m, overlap=overlap, apply_rope=False)
    np.testing.assert_allclose(pool, pool2, atol=1e-14)


def test_compress_trailing_partial_window_is_not_an_entry():
    x = np.random.default_rng(2).standard_normal((1, 11, 3))
    assert O.compress(x, None, None, None, m=4, overlap=1, apply_rope=False).shape == (1, 2, 3)


def test_compress_m1_is_identity_plus_rope():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 9, 10))
    z = rng.standard_normal((1, 9, 10))
    pos = np.arange(9)[None] + 5
    pool = O.compress(x, z, None, pos, m=1, overlap=0, apply_rope=True, R=4, theta=100.0)
    np.testing.assert_allclose(pool, _rope_complex(x, pos, 4, 100.0), atol=1e-13)


def test_compress_single_window_is_global_mean():
    x = np.random.default_rng(4).standard_normal((1, 32, 5))
    pool = O.compress(x, None, None, None, m=32, overlap=0, apply_rope=False)
    np.testing.assert_allclose(pool[0, 0], x[0].mean(axis=0), atol=1e-14)


@pytest.mark.parametrize("overlap", [0, 1])
def test_compress_gate_selects_and_slot_bias_alignment(overlap):
    rng = np.random.default_rng(5)
    S, c, m = 24, 4, 4
    x = rng.standard_normal((1, S, c))
    # a dominant token logit makes the entry that token's row
    z = np.zeros((1, S, c))
    z[0, 13, :] = 800.0
    pool = O.compress(x, z, None, None, m=m, overlap=overlap, apply_rope=False)
    owners = [w for w in range(S // m)
              if ((w - 1) * m if overlap else w * m) <= 13 < (w + 1) * m]
    for w in owners:
        np.testing.assert_allclose(pool[0, w], x[0, 13], atol=1e-12)
    # a dominant bias on slot s makes entry w the row of token (first token of window)+s
    Lw = 2 * m if overlap else m
    for s in range(Lw):
        bias = np.zeros((Lw, c))
        bias[s] = 800.0
        pool = O.compress(x, None, bias, None, m=m, overlap=overlap, apply_rope=False)
        for w in range(1, S // m):
            lo = (w - 1) * m if overlap else w * m
            np.testing.assert_allclose(pool[0, w], x[0, lo + s], atol=1e-12)
    # entry 0 with overlap: the older half is missing, slots m..2m-1 hold tokens 0..m-1
    if overlap:
        bias = np.zeros((Lw, c))
        bias[m + 2] = 800.0
        pool = O.compress(x, None, bias, None, m=m, overlap=1, apply_rope=False)
        np.testing.assert_allclose(pool[0, 0], x[0, 2], atol=1e-12)


def test_compress_rope_position_is_first_token_of_own_block():
    rng = np.random.default_rng(6)
    S, c, m, R = 16, 8, 4, 4
    x = rng.standard_normal((1, S, c))
    pos = (np.arange(S) * 3 + 11)[None]
    plain = O.compress(x, None, None, None, m=m, overlap=1, apply_rope=False)
    roped = O.compress(x, None, None, pos, m=m, overlap=1, apply_rope=True, R=R, theta=50.0)
    for w in range(S // m):
        np.testing.assert_allclose(roped[0, w], _rope_complex(plain[0, w], pos[0, w * m], R, 50.0),
                                   atol=1e-13)


# ---------------------------------------------------------------- indexer / top-k
def test_indexer_hand_example():
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([2.0, -1.0])
    keys = np.array([[1.0, 1.0], [-1.0, 2.0], [3.0, -1.0]])
    # head 0 dots [1,-1,3] -> relu [1,0,3]; head 1 dots [1,2,-1] -> relu [1,2,0]
    np.testing.assert_allclose(O.indexer_scores_row(q, w, keys, 3), [1.0, -2.0, 6.0], atol=0)
    np.testing.assert_allclose(O.indexer_scores_row(q, w, keys, 2), [1.0, -2.0], atol=0)


def test_indexer_topk_invariant_to_positive_scaling():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((4, 16))
    w = rng.standard_normal(4)
    keys = rng.standard_normal((50, 16))
    base = O.topk_select_row(O.indexer_scores_row(q, w, keys, 50), 10)[0]
    assert O.topk_select_row(O.indexer_scores_row(q * 3.0, w, keys, 50), 10)[0] == base
    assert O.topk_select_row(O.indexer_scores_row(q, w * 0.25, keys, 50), 10)[0] == base
    # one head with unit weight ranks entries by their positive dot products
    s1 = O.indexer_scores_row(q[:1], np.ones(1), keys, 50)
    d = keys @ q[0]
    assert np.all(s1 == np.maximum(d, 0))


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    vis = int(rng.integers(0, 40))
    K = int(rng.integers(1, 20))
    scores = rng.integers(-3, 4, size=vis).astype(np.float64)  # many exact ties
    ranked, padded = O.topk_select_row(scores, K)
    brute = sorted(range(vis), key=lambda i: (-scores[i], i))[: min(K, vis)]
    assert ranked == brute
    assert list(padded[: len(brute)]) == brute and all(p == -1 for p in padded[len(brute):])


# ---------------------------------------------------------------- attention row
def test_sink_is_an_extra_logit_with_zero_value():
    rng = np.random.default_rng(8)
    H, Nk, D, dv = 3, 7, 6, 6
    q, keys, sink = rng.standard_normal((H, D)), rng.standard_normal((Nk, D)), rng.standard_normal(H)
    o = O.attend_row(q, keys, sink, 0.4, dv)
    for h in range(H):
        lg = np.concatenate([0.4 * keys @ q[h], [sink[h]]])
        p = np.exp(lg - logsumexp(lg))
        vals = np.concatenate([keys[:, :dv], np.zeros((1, dv))])
        np.testing.assert_allclose(o[h], p @ vals, atol=1e-14)
    # sink -> -inf is plain softmax attention
    o_inf = O.attend_row(q, keys, np.full(H, -1e300), 0.4, dv)
    lg = 0.4 * q @ keys.T
    p = np.exp(lg - logsumexp(lg, axis=1, keepdims=True))
    np.testing.assert_allclose(o_inf, p @ keys[:, :dv], atol=1e-14)


def test_single_key_closed_form():
    rng = np.random.default_rng(9)
    q, k, s = rng.standard_normal((2, 5)), rng.standard_normal((1, 5)), np.array([0.3, -1.2])
    o = O.attend_row(q, k, s, 0.7, 3)
    for h in range(2):
        l = 0.7 * q[h] @ k[0]
        np.testing.assert_allclose(o[h], k[0, :3] * expit(l - s[h]), atol=1e-15)
    assert np.all(O.attend_row(q, k[:0], s, 0.7, 3) == 0)


def test_shared_kv_derivative():
    """K=V: moving one key channel moves both its logit and its value contribution.

    d o_h / d k_j[d] = p_j e_d + scale q_h[d] p_j (v_j - o_h)   (d < dv)
    d o_h / d k_j[d] = scale q_h[d] p_j (v_j - o_h)             (d >= dv)
    """
    rng = np.random.default_rng(10)
    H, Nk, D, dv, sc = 2, 5, 6, 4, 0.8
    q, keys, sink = rng.standard_normal((H, D)), rng.standard_normal((Nk, D)), rng.standard_normal(H)
    o = O.attend_row(q, keys, sink, sc, dv)
    lg = sc * q @ keys.T
    mx = np.maximum(lg.max(1), sink)
    e = np.exp(lg - mx[:, None])
    p = e / (e.sum(1) + np.exp(sink - mx))[:, None]
    eps = 1e-6
    for j in range(Nk):
        for d in range(D):
            kp, km = keys.copy(), keys.copy()
            kp[j, d] += eps
            km[j, d] -= eps
            num = (O.attend_row(q, kp, sink, sc, dv) - O.attend_row(q, km, sink, sc, dv)) / (2 * eps)
            ed = np.zeros(dv)
            if d < dv:
                ed[d] = 1.0
            ana = p[:, j, None] * ed[None] + sc * q[:, d, None] * p[:, j, None] * (keys[j, :dv] - o)
            np.testing.assert_allclose(num, ana, atol=1e-7)


# ---------------------------------------------------------------- full layers
def _tiny_inputs(seed, S=48, H=3, D=16, R=8, cI=8, nI=2, m=4, overlap=1):
    rng = np.random.default_rng(seed)
    Lw = 2 * m if overlap else m
    return dict(
        q=rng.standard_normal((1, S, H, D)), kv=rng.standard_normal((1, S, D)),
        z=rng.standard_normal((1, S, D)), bias=0.1 * rng.standard_normal((Lw, D)),
        qI=rng.standard_normal((1, S, nI, cI)), wI=rng.standard_normal((1, S, nI)),
        kI=rng.standard_normal((1, S, cI)), zI=rng.standard_normal((1, S, cI)),
        biasI=0.1 * rng.standard_normal((Lw, cI)), sink=rng.standard_normal(H),
        pos=np.arange(S)[None].astype(np.int64))


def _dense_reference(q, kv, pool, sink, pos, *, n_win, m, scale, dv, R, theta, rotate_out):
    """Dense attention with the concatenated mask [sliding_causal | block_bias] and a sink column.

    Built as the "Attention mask layout" section describes: keys are the S token rows
    (rotated at their positions) followed by the P pool entries; the sliding section lets
    query t see (t-n_win, t]; the compressor section lets it see entry w iff w < (t+1)//m.
    """
    S, H, D = q.shape[1], q.shape[2], q.shape[3]
    P = pool.shape[1]
    keys = np.concatenate([_rope_complex(kv[0], pos[0], R, theta), pool[0]], axis=0)
    out = np.zeros((S, H, dv))
    for t in range(S):
        mask = np.full(S + P, -np.inf)
        mask[max(0, t - n_win + 1):t + 1] = 0.0
        mask[S:S + (t + 1) // m] = 0.0
        qt = _rope_complex(q[0, t], pos[0, t], R, theta)
        lg = scale * qt @ keys.T + mask[None]
        lg = np.concatenate([lg, sink[:, None]], axis=1)
        p = np.exp(lg - logsumexp(lg, axis=1, keepdims=True))
        o = p[:, :-1] @ keys[:, :dv]
        if rotate_out:
            o = _rope_complex(o, pos[0, t], R, theta, sign=-1.0)
        out[t] = o
    return out


def test_hca_equals_dense_masked_attention():
    x = _tiny_inputs(11, S=40, m=8, overlap=0)
    kw = dict(m=8, n_win=6, scale=0.3, dv=16, R=8, theta=1000.0, rotate_out=1)
    res = O.hca_layer(x["q"], x["kv"], x["z"], x["bias"], x["sink"], x["pos"], **kw)
    ref = _dense_reference(x["q"], x["kv"], res["pool"], x["sink"], x["pos"], **kw)
    np.testing.assert_allclose(res["out"][0], ref, atol=1e-12)


def test_sliding_layer_equals_dense_window_attention():
    """The window-only layer is the dense masked attention with an empty compressor section."""
    x = _tiny_inputs(15, S=40)
    kw = dict(n_win=7, scale=0.3, dv=16, R=8, theta=1000.0, rotate_out=1)
    res = O.sliding_layer(x["q"], x["kv"], x["sink"], x["pos"], **kw)
    ref = _dense_reference(x["q"], x["kv"], np.zeros((1, 0, 16)), x["sink"], x["pos"], m=1, **kw)
    np.testing.assert_allclose(res["out"][0], ref, atol=1e-12)
    # the first query sees only itself: softmax of one logit against the sink
    qt = _rope_complex(x["q"][0, 0], 0, 8, 1000.0)
    lg = 0.3 * qt @ x["kv"][0, 0]
    p = 1.0 / (1.0 + np.exp(x["sink"] - lg))
    np.testing.assert_allclose(res["out"][0, 0], p[:, None] * x["kv"][0, 0][None, :16], atol=1e-12)


def test_sliding_layer_follows_the_worked_mask():
    """Keys of the sliding layer = the [sliding] grid of the worked 16-token example (window 8),
    attended with the sink as an extra logit and the output rotated back by -t."""
    g = _read_golden_sections("mask_example_16tok.txt")
    x = _tiny_inputs(16, S=16)
    R, theta, scale = 8, 1000.0, 0.4
    res = O.sliding_layer(x["q"], x["kv"], x["sink"], x["pos"], n_win=8, scale=scale, dv=16, R=R, theta=theta,
                          rotate_out=1)
    keys = _rope_complex(x["kv"][0], x["pos"][0], R, theta)
    for t in range(16):
        vis = [j for j in range(16) if g["sliding"][t][j] == "1"]
        qt = _rope_complex(x["q"][0, t], x["pos"][0, t], R, theta)
        lg = scale * qt @ keys[vis].T
        mx = np.maximum(lg.max(axis=1), x["sink"])
        e = np.exp(lg - mx[:, None])
        o = (e @ keys[vis]) / (e.sum(axis=1) + np.exp(x["sink"] - mx))[:, None]
        np.testing.assert_allclose(res["out"][0, t], _rope_complex(o, x["pos"][0, t], R, theta, sign=-1.0),
                                   atol=1e-12)


def test_csa_with_topk_covering_pool_equals_dense_masked_attention():
    x = _tiny_inputs(12, S=48, m=4, overlap=1)
    kw = dict(m=4, n_win=5, scale=0.3, dv=16, R=8, theta=1000.0, rotate_out=1)
    res = O.csa_layer(x["q"], x["kv"], x["z"], x["bias"], x["qI"], x["wI"], x["kI"], x["zI"],
                      x["biasI"], x["sink"], x["pos"], overlap=1, topk=12, **kw)
    assert res["pool"].shape[1] == 12
    ref = _dense_reference(x["q"], x["kv"], res["pool"], x["sink"], x["pos"], **kw)
    np.testing.assert_allclose(res["out"][0], ref, atol=1e-12)
    # queries t < m-1 select nothing
    assert np.all(res["idx"][0, :3] == -1)


def test_csa_topk_subset_differs_from_dense():
    # with K < P the indexer really prunes: some rows must differ from the dense result
    x = _tiny_inputs(13, S=48)
    kw = dict(m=4, n_win=3, scale=1.0, dv=16, R=8, theta=1000.0, rotate_out=1)
    res = O.csa_layer(x["q"], x["kv"], x["z"], x["bias"], x["qI"], x["wI"], x["kI"], x["zI"],
                      x["biasI"], x["sink"], x["pos"], overlap=1, topk=2, **kw)
    ref = _dense_reference(x["q"], x["kv"], res["pool"], x["sink"], x["pos"], **kw)
    assert np.abs(res["out"][0] - ref).max() > 1e-3
    # rows with at most two visible entries keep everything and match exactly
    np.testing.assert_allclose(res["out"][0, :11], ref[:11], atol=1e-12)


@pytest.mark.parametrize("delta", [1, 1000, 65536])
def test_outputs_invariant_to_uniform_position_shift(delta):
    x = _tiny_inputs(14, S=40)
    kw = dict(m=4, overlap=1, n_win=6, topk=3, scale=0.5, dv=16, R=8, theta=160000.0,
              rotate_out=1)
    a = O.csa_layer(x["q"], x["kv"], x["z"], x["bias"], x["qI"], x["wI"], x["kI"], x["zI"],
                    x["biasI"], x["sink"], x["pos"], **kw)
    b = O.csa_layer(x["q"], x["kv"], x["z"], x["bias"], x["qI"], x["wI"], x["kI"], x["zI"],
                    x["biasI"], x["sink"], x["pos"] + delta, **kw)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], atol=1e-10)
    # without the -i output rotation the shift shows up in the rope slice
    kw["rotate_out"] = 0
    a = O.csa_layer(x["q"], x["kv"], x["z"], x["bias"], x["qI"], x["wI"], x["kI"], x["zI"],
                    x["biasI"], x["sink"], x["pos"], **kw)
    b = O.csa_layer(x["q"], x["kv"], x["z"], x["bias"], x["qI"], x["wI"], x["kI"], x["zI"],
                    x["biasI"], x["sink"], x["pos"] + delta, **kw)
    assert np.abs(a["out"][..., -8:] - b["out"][..., -8:]).max() > 1e-6
    np.testing.assert_allclose(a["out"][..., :-8], b["out"][..., :-8], atol=1e-10)


def test_output_rotation_single_self_key_closed_form():
    """One key (the query's own token, window 1, nothing pooled yet): the rotated-back
    output is sigmoid(l - s) times the UNROTATED key row."""
    rng = np.random.default_rng(15)
    H, D, R = 2, 12, 4
    q = rng.standard_normal((1, 1, H, D))
    kv = rng.standard_normal((1, 1, D))
    sink = rng.standard_normal(H)
    pos = np.array([[777]])
    kv_rot = O.rope_rotate(kv, pos, R, 10.0)
    out = O.sparse_mqa_attention(q, kv_rot, np.zeros((1, 0, D)), None, sink, pos,
                                 np.array([[0]]), n_win=1, m=4, scale=0.5, dv=D, R=R,
                                 theta=10.0, rope_q=True, rotate_out=True)
    for h in range(H):
        l = 0.5 * q[0, 0, h] @ kv[0, 0]  # rotation by the same angle cancels in the logit
        np.testing.assert_allclose(out[0, 0, h], kv[0, 0] * expit(l - sink[h]), atol=1e-14)


def test_no_keys_gives_zero_output():
    q = np.ones((1, 1, 2, 4))
    out = O.sparse_mqa_attention(q, np.zeros((1, 1, 4)), np.zeros((1, 4, 4)), None, np.zeros(2),
                                 np.array([[0]]), np.array([[0]]), n_win=0, m=4, scale=1.0,
                                 dv=4, R=2, theta=10.0, rope_q=True, rotate_out=True)
    assert np.all(out == 0)


def test_ring_window_matches_linear_window():
    rng = np.random.default_rng(16)
    S, D, H, ring, n_win = 50, 8, 2, 8, 6
    kv = rng.standard_normal((1, S, D))
    pool = rng.standard_normal((1, S // 4, D))
    q = rng.standard_normal((1, 1, H, D))
    sink = rng.standard_normal(H)
    t = 45
    ringbuf = np.zeros((1, ring, D))
    for j in range(S):  # a ring keeps the latest `ring` rows
        ringbuf[0, j % ring] = kv[0, j] if j <= t else ringbuf[0, j % ring]
    idx = np.array([[[3, 7, 1, -1]]])
    kw = dict(n_win=n_win, m=4, scale=0.4, dv=D, R=4, theta=99.0, rope_q=False, rotate_out=False)
    a = O.sparse_mqa_attention(q, kv, pool, idx, sink, np.array([[t]]), np.array([[t]]), **kw)
    b = O.sparse_mqa_attention(q, ringbuf, pool, idx, sink, np.array([[t]]), np.array([[t]]),
                               win_ring=ring, **kw)
    np.testing.assert_allclose(a, b, atol=0)


def test_dsa_token_level_includes_self():
    # m=1, no window: query t sees tokens j <= t through the (identity) pool
    rng = np.random.default_rng(17)
    S, D, H = 6, 8, 2
    pool = rng.standard_normal((1, S, D))
    q = rng.standard_normal((1, S, H, D))
    sink = np.full(H, -1e300)
    qi = np.arange(S)[None]
    out = O.sparse_mqa_attention(q, np.zeros((1, S, D)), pool, None, sink, qi, qi, n_win=0, m=1,
                                 scale=1.0, dv=D, R=2, theta=10.0, rope_q=False, rotate_out=False)
    np.testing.assert_allclose(out[0, 0], np.tile(pool[0, 0], (H, 1)), atol=1e-14)


# ---------------------------------------------------------------- decode cache
@pytest.mark.parametrize("m,overlap", [(4, True), (8, False), (1, False)])
def test_decode_append_matches_prefill_compression(m, overlap):
    """Appending tokens one at a time through the decode cache ("Cache layers": window ring
    and compressor buffer with its overlap state) gives the pool that compressing the
    whole prefix at once gives, and a window ring holding the last rows rotated at their
    positions; entries past the pool capacity are not written, and a partial last block
    is not an entry."""
    rng = np.random.default_rng(11)
    S, c, R, ring = 37, 16, 8, 16
    lw = 2 * m if overlap else m
    x = rng.standard_normal((1, S, c))
    z = rng.standard_normal((1, S, c))
    bias = 0.3 * rng.standard_normal((lw, c))
    pos = (np.arange(S) * 3 + 1000)[None]            # positions are not the cache indices
    batch = O.compress(x, z, bias, pos, m=m, overlap=overlap, apply_rope=True, R=R, theta=10000.0)
    P_cap = S // m - 1                                # the last complete entry does not fit
    cache = O.new_decode_cache(c, m=m, overlap=overlap, P_cap=P_cap, win_ring=ring)
    for t in range(S):
        O.decode_append(cache, x[0, t], z[0, t], pos[0, t], t, m=m, overlap=overlap, bias=bias,
                        apply_rope=True, R=R, theta=10000.0)
    np.testing.assert_allclose(cache["pool"], batch[0, :P_cap], rtol=0, atol=1e-12)
    rot = O.rope_rotate(x, pos, R, 10000.0)
    for j in range(S - ring, S):
        np.testing.assert_allclose(cache["win"][j % ring], rot[0, j], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariants
def test_attention_is_invariant_to_the_order_of_the_index_list():
    """Attention is a sum over a key set: any order of the selected entries (and of the -1
    holes among them) gives the same output."""
    x = _tiny_inputs(17, S=40)
    kw = dict(n_win=5, m=4, scale=0.3, dv=16, R=8, theta=1000.0, rope_q=True, rotate_out=1)
    pool = O.compress(x["kv"], x["z"], x["bias"], x["pos"], m=4, overlap=True, apply_rope=True, R=8, theta=1000.0)
    kv_rot = O.rope_rotate(x["kv"], x["pos"], 8, 1000.0)
    qi = np.arange(40)[None]
    idx = O.indexer_topk(x["qI"], x["wI"], O.compress(x["kI"], x["zI"], x["biasI"], x["pos"], m=4, overlap=True,
                                                        apply_rope=False), qi, m=4, topk=5)
    rng = np.random.default_rng(0)
    shuffled = np.stack([np.stack([rng.permutation(r) for r in idx[0]])])
    a = O.sparse_mqa_attention(x["q"], kv_rot, pool, idx, x["sink"], x["pos"], qi, **kw)
    b = O.sparse_mqa_attention(x["q"], kv_rot, pool, shuffled, x["sink"], x["pos"], qi, **kw)
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_compress_is_linear_in_the_rows_and_its_weights_sum_to_one():
    """For fixed logits the pool is a per-channel convex combination of the window's rows:
    linear in the rows (RoPE included), and constant rows pool to that constant."""
    x = _tiny_inputs(18, S=32)
    kw = dict(m=4, overlap=True, apply_rope=True, R=8, theta=1000.0)
    y = np.random.default_rng(1).standard_normal(x["kv"].shape)
    lhs = O.compress(2.0 * x["kv"] - 3.0 * y, x["z"], x["bias"], x["pos"], **kw)
    rhs = 2.0 * O.compress(x["kv"], x["z"], x["bias"], x["pos"], **kw) - 3.0 * O.compress(y, x["z"], x["bias"],
                                                                                          x["pos"], **kw)
    np.testing.assert_allclose(lhs, rhs, atol=1e-12)
    const = np.broadcast_to(np.linspace(-1.0, 1.0, 16), x["kv"].shape).copy()
    pooled = O.compress(const, x["z"], x["bias"], x["pos"], m=4, overlap=True, apply_rope=False)
    np.testing.assert_allclose(pooled, const[:, :pooled.shape[1]], atol=1e-12)  # every row is the same vector


# ---------------------------------------------------------------- grouped output projection
def _grouped_inputs(seed, T=5, H=8, dv=6, g=4, dg=3, hidden=7):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, H, dv)), rng.standard_normal((g, dg, (H // g) * dv)),
            rng.standard_normal((hidden, g * dg)))


def test_grouped_out_proj_equals_dense_block_diagonal_product():
    """o_a_proj as one dense product with a block-diagonal weight (block i maps the flattened
    heads of group i to its d_g outputs), then o_b_proj: written out element by element."""
    o, wa, wb = _grouped_inputs(0)
    T, H, dv = o.shape
    g, dg, width = wa.shape
    y = O.grouped_out_proj(o, wa, wb)
    ref = np.zeros((T, wb.shape[0]))
    for t in range(T):
        flat = o[t].reshape(H * dv)
        u = np.zeros(g * dg)
        for i in range(g):
            for r in range(dg):
                u[i * dg + r] = sum(wa[i, r, c] * flat[i * width + c] for c in range(width))
        ref[t] = [sum(wb[k, j] * u[j] for j in range(g * dg)) for k in range(wb.shape[0])]
    np.testing.assert_allclose(y, ref, atol=1e-12)


def test_grouped_out_proj_special_cases():
    o, wa, wb = _grouped_inputs(1)
    T, H, dv = o.shape
    # one group: the plain low-rank product wb @ wa @ flat(o)
    wa1 = np.random.default_rng(2).standard_normal((1, 5, H * dv))
    wb1 = np.random.default_rng(3).standard_normal((7, 5))
    np.testing.assert_allclose(O.grouped_out_proj(o, wa1, wb1), o.reshape(T, -1) @ wa1[0].T @ wb1.T, atol=1e-12)
    # identity projections give back the flattened heads
    g = 4
    eye_a = np.stack([np.eye((H // g) * dv)] * g)
    np.testing.assert_allclose(O.grouped_out_proj(o, eye_a, np.eye(H * dv)), o.reshape(T, -1), atol=1e-12)
    # heads of one group only reach that group's channels of the intermediate
    o2 = np.zeros_like(o)
    o2[:, 2:4] = o[:, 2:4]            # heads 2 and 3 = group 1 of 4
    u = O.grouped_out_proj(o2, wa, np.eye(wb.shape[1]))
    dg = wa.shape[1]
    assert np.abs(u[:, dg:2 * dg]).max() > 0 and np.abs(np.delete(u, np.s_[dg:2 * dg], axis=1)).max() == 0


# ---------------------------------------------------------------- storage rounding
def test_store_as_bf16_rounds_to_nearest_even():
    """bf16 storage (7 explicit mantissa bits) of values worked out by hand: exact ties go to
    the even neighbour (also across a binade edge and in the subnormal range), values past a
    tie round away, signs and zeros are kept, and a float32 above the bf16 range overflows."""
    p = 2.0 ** -8
    cases = [
        (1.0 + p, 1.0),                          # tie between 1 and 1 + 2^-7: even is 1
        (1.0 + 3 * p, 1.0 + 2.0 ** -6),          # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
        (-(1.0 + p), -1.0),                      # the negative tie
        (1.0 + p + 2.0 ** -20, 1.0 + 2.0 ** -7),  # just past the tie
        (1.0 + p - 2.0 ** -20, 1.0),             # just below it
        (2.0 - p, 2.0),                          # tie at the top of a binade carries into the exponent
        (2.0 - 3 * 2.0 ** -9, 2.0 - 2.0 ** -7),  # below that tie
        (0.1, 0.10009765625),                    # 0x3DCCCCCD -> 0x3DCD
        ((2.0 - 2.0 ** -7) * 2.0 ** 127, (2.0 - 2.0 ** -7) * 2.0 ** 127),  # largest finite bf16
        (float(np.finfo(np.float32).max), math.inf),  # above bf16's range: rounds to infinity
        (2.0 ** -133, 2.0 ** -133),              # smallest bf16 subnormal
        (2.0 ** -134, 0.0),                      # tie between 0 and it: even is 0
        (3 * 2.0 ** -134, 2.0 ** -132),          # tie between 2^-133 (odd) and 2^-132 (even)
        (5.0, 5.0), (-7.5, -7.5),                # exactly representable values are unchanged
    ]
    got = O.store_as(np.array([c[0] for c in cases]), "bf16")
    for (x, want), g in zip(cases, got):
        assert g == want, f"store_as({x!r}, 'bf16') = {g!r}, expected {want!r}"
    zeros = O.store_as(np.array([0.0, -0.0]), "bf16")
    assert np.all(zeros == 0.0) and not np.signbit(zeros[0]) and np.signbit(zeros[1])


def test_store_as_matches_library_conversions():
    """bf16 storage equals torch's float32 -> bfloat16 conversion (round to nearest even) on a
    grid of random values over many binades, with exact ties planted; f32 storage equals
    numpy's float32 cast; no storage keeps float64."""
    import torch
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200000) * np.exp2(rng.integers(-140, 120, 200000))).astype(np.float32)
    u = x.view(np.uint32)
    u[::5] = (u[::5] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)   # exact ties
    u[1::5] = (u[1::5] & np.uint32(0xFFFF0000)) | np.uint32(0x7FFF)  # just below a tie
    u[2::5] = (u[2::5] & np.uint32(0xFFFF0000)) | np.uint32(0x8001)  # just above a tie
    x = u.view(np.float32)
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.store_as(x.astype(np.float64), "bf16")
    np.testing.assert_array_equal(got, want)
    y = rng.standard_normal(1000) * 1e3
    np.testing.assert_array_equal(O.store_as(y, "f32"), y.astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(O.store_as(y, None), y)
