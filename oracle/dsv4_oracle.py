"""Plain fp64 CPU oracle for the DeepSeek-V4 hybrid compressed attention core.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or call it.  It shares no
code, header, table or helper with the CUDA library; the two meet only through
the seeded input generator in ``synth/`` (which holds no arithmetic of the
method).

Every step widens its inputs exactly to float64 and computes in float64, one
query row or one pool entry at a time, in the order the method states it.
Library primitives used as steps: ``numpy`` matrix products, ``exp``, ``cos``,
``sin`` and ``lexsort``.  There is no blocking, fusion or reordering.

Sources (HF Transformers model docs):
  [V4]   "DeepSeek-V4" doc, section "Architecture (paper §2)" → "Hybrid
         attention (§2.3)", "Attention mask layout", "Cache layers", and the
         ``DeepseekV4Config`` parameter list.
  [V32]  "DeepSeek-V3.2" doc, section "DeepSeek Sparse Attention (DSA)" and
         the ``DeepseekV32Config`` parameter list.

The pages name the equations (indexer eqs. 13-17, output rotation eq. 26, sink
eq. 27) but never print them, and give no pooling formula for the compressor.
Where they are silent this oracle takes the readings below; each is listed with
its status:

  R1 compressor window (overlap): entry w pools tokens [(w-1)m, (w+1)m) clipped
     at 0 (CSA); [wm, (w+1)m) without overlap (HCA).  Pinned only through the
     visibility rule it implies (entry w closes at token (w+1)m-1).
  R2 compressor weights: per-channel softmax over the window of
     (token logit + per-slot bias), weighted sum of the rows.
     PARITY UNPINNED against the method (the pages print no formula); pinned
     against its own closed forms (mean pooling, identity at m=1, one-hot gate).
  R3 entry RoPE position = position of the first token of the entry's own
     block; indexer keys carry no RoPE.  PARITY UNPINNED against the method.
  R4 indexer score I[t,w] = sum_h wI[t,h] * relu(qI[t,h] . kI_w).  The ReLU
     gate is a reading (DSA-style); PARITY UNPINNED against the method.
  R5 sink = one extra logit s_h in the softmax denominator with a zero value
     row (eq. 27 as the pages name it).  Pinned (closed forms).
  R6 output rotation: the rope slice of the output is rotated by -qpos (eq. 26)
     when the value width equals head_dim.  Pinned (shift invariance).
  R7 DSA (m=1, no window): a query sees tokens j <= t (itself included).
  R13 sliding-window layers (`sliding_attention`): no pool and no indexer; keys
     are the window rows only; their RoPE base is rope_theta (10000), since
     compress_rope_theta belongs to the compressed layers.  Pinned (dense masked
     attention with an empty compressor section).
  R14 grouped output projection: head group i = the contiguous heads [iH/g, (i+1)H/g),
     concatenated in head order and projected by its own o_a_proj weight; the
     groups' results, concatenated in group order, feed o_b_proj.  No biases
     (attention_bias=False).  PARITY UNPINNED against the method (the pages give
     the shapes only); pinned against its own closed forms.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "store_as",
    "rope_rotate",
    "pool_window",
    "compress",
    "visible_entries",
    "window_tokens",
    "indexer_scores_row",
    "topk_select_row",
    "attend_row",
    "sparse_mqa_attention",
    "indexer_topk",
    "csa_layer",
    "hca_layer",
    "sliding_layer",
    "grouped_out_proj",
    "new_decode_cache",
    "decode_append",
]


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def store_as(a, store):
    """Round float64 values to the storage dtype the caller keeps them in.

    store=None keeps float64; "f32" rounds to float32; "bf16" rounds to the nearest
    bfloat16 (ties to even), as a cache of bf16 rows would.  Decisions taken on stored
    values (top-k over indexer scores of a bf16 key pool) are then taken on the same
    values the kernels read.
    """
    if store is None:
        return _f64(a)
    f = np.asarray(a, dtype=np.float32)
    if store == "f32":
        return f.astype(np.float64)
    assert store == "bf16", store
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# RoPE  [V4] "Hybrid attention (§2.3)": partial interleaved-pair rotary
# embedding on the trailing qk_rope_head_dim channels of each head;
# ``partial_rotary_factor`` in DeepseekV4Config; ``rope_theta`` /
# ``compress_rope_theta`` give the base.
# --------------------------------------------------------------------------
def rope_rotate(x, pos, R, theta, sign=1.0):
    """Rotate the trailing R channels of ``x`` as R/2 interleaved pairs.

    Pair k is channels (c-R+2k, c-R+2k+1); its angle is sign * pos * theta^(-2k/R)
    and (a, b) -> (a cos - b sin, a sin + b cos).  ``pos`` broadcasts against
    ``x.shape[:-1]``.  sign=-1 gives the inverse rotation used on the output
    (eq. 26, rotation by position -i).
    """
    x = _f64(x)
    out = x.copy()
    if R == 0:
        return out
    c = x.shape[-1]
    k = np.arange(R // 2, dtype=np.float64)
    inv_freq = float(theta) ** (-2.0 * k / R)
    ang = sign * np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    cos, sin = np.cos(ang), np.sin(ang)
    a = x[..., c - R::2]
    b = x[..., c - R + 1::2]
    out[..., c - R::2] = a * cos - b * sin
    out[..., c - R + 1::2] = a * sin + b * cos
    return out


# --------------------------------------------------------------------------
# KV compressor  [V4] "Hybrid attention (§2.3)" CSA item (low-compression pool,
# m=4, overlapping windows) and HCA item (m'=128, non-overlapping);
# "Cache layers" (CSA keeps overlap state, HCA does not); ``compress_rates``.
# --------------------------------------------------------------------------
def pool_window(w, m, overlap, S):
    """Tokens feeding pool entry w and their slot numbers (reading R1).

    overlap: tokens [(w-1)m, (w+1)m) clipped to [0, S); slot = j - (w-1)m in [0, 2m).
    otherwise: tokens [wm, (w+1)m); slot = j - wm in [0, m).
    """
    lo = (w - 1) * m if overlap else w * m
    hi = (w + 1) * m
    js = [j for j in range(lo, hi) if 0 <= j < S]
    return js, [j - lo for j in js]


def compress(x, z, bias, pos, *, m, overlap, apply_rope, R=0, theta=160000.0):
    """Pool [B,S,c] token rows into [B, S//m, c] entries (readings R1-R3).

    entry_w[d] = sum_{j in J_w} alpha_j[d] x_j[d],
    alpha_.[d] = softmax over j in J_w of (z_j[d] + bias[slot(j), d]).
    ``z`` (per-token compressor logits, [B,S,c]) and ``bias`` (per-slot, [2m or m, c])
    may be None (= 0).  With ``apply_rope`` the entry's trailing R channels are
    rotated at pos[b, w*m] (reading R3).
    """
    x = _f64(x)
    z = _f64(z)
    bias = _f64(bias)
    B, S, c = x.shape
    P = S // m
    out = np.zeros((B, P, c))
    for b in range(B):
        for w in range(P):
            js, slots = pool_window(w, m, overlap, S)
            logit = np.zeros((len(js), c))
            if z is not None:
                logit = logit + z[b, js]
            if bias is not None:
                logit = logit + bias[slots]
            mx = logit.max(axis=0)
            e = np.exp(logit - mx)
            alpha = e / e.sum(axis=0)
            entry = (alpha * x[b, js]).sum(axis=0)
            if apply_rope:
                entry = rope_rotate(entry, pos[b, w * m], R, theta)
            out[b, w] = entry
    return out


# --------------------------------------------------------------------------
# Visibility  [V4] "Attention mask layout": HCA query t sees entry w iff
# w < (t+1)//m; CSA queries before the first window closes (t < m-1) get
# nothing (-1 sentinels); the sliding section is the causal window of
# ``sliding_window`` tokens.  [V32] DSA: "previous tokens" (reading R7).
# --------------------------------------------------------------------------
def visible_entries(t, m, P_cap=None):
    v = (t + 1) // m
    return v if P_cap is None else min(v, P_cap)


def window_tokens(t, n_win):
    """Cache indices of the sliding-window keys of a query at cache index t."""
    return list(range(max(0, t - n_win + 1), t + 1))


# --------------------------------------------------------------------------
# Lightning Indexer  [V4] CSA item ("Lightning Indexer (eqs. 13-17)"),
# ``index_n_heads`` (eq. 14), ``index_head_dim``, ``index_topk`` (eq. 17);
# [V32] DSA item 1 (low head count, per-head ``weights_proj``; Hadamard is
# orthogonal so scores are computed directly) and item 2 (top-k selection).
# --------------------------------------------------------------------------
def indexer_scores_row(qI_t, wI_t, poolI, vis):
    """I[w] = sum_h wI[h] * relu(qI[h] . poolI[w]) for w < vis (reading R4)."""
    qI_t = _f64(qI_t)
    wI_t = _f64(wI_t)
    keys = _f64(poolI)[:vis]
    dots = keys @ qI_t.T  # [vis, nI]
    return (np.maximum(dots, 0.0) * wI_t[None, :]).sum(axis=1)


def topk_select_row(scores, K):
    """Rank visible entries by (score desc, index asc); keep the first min(K, vis).

    Returns (ranked_indices, padded) where padded has length K with -1 sentinels
    after the selected entries ([V4] "Attention mask layout", CSA item).
    Ties: the lower index wins.
    """
    scores = np.asarray(scores, dtype=np.float64)
    vis = scores.shape[0]
    order = np.lexsort((np.arange(vis), -scores))
    ranked = [int(w) for w in order[: min(K, vis)]]
    padded = np.full(K, -1, dtype=np.int64)
    padded[: len(ranked)] = ranked
    return ranked, padded


def indexer_topk(qI, wI, poolI, q_index, *, m, topk, P_cap=None, rows=None,
                 return_scores=False):
    """Scores and top-k for every (b, s) query (or the listed rows).

    qI [B,Sq,nI,cI], wI [B,Sq,nI], poolI [B,P,cI], q_index [B,Sq] cache indices.
    Returns idx [B,Sq,topk] int64 in rank order (-1 padded) for the computed rows
    (others -2), and optionally a dict {(b,s): scores}.
    """
    B, Sq = qI.shape[0], qI.shape[1]
    P = poolI.shape[1] if P_cap is None else P_cap
    idx = np.full((B, Sq, topk), -2, dtype=np.int64)
    all_scores = {}
    if rows is None:
        rows = [(b, s) for b in range(B) for s in range(Sq)]
    for b, s in rows:
        vis = visible_entries(int(q_index[b, s]), m, P)
        sc = indexer_scores_row(qI[b, s], wI[b, s], poolI[b], vis)
        _, idx[b, s] = topk_select_row(sc, topk)
        if return_scores:
            all_scores[(b, s)] = sc
    return (idx, all_scores) if return_scores else idx


# --------------------------------------------------------------------------
# Core attention  [V4] "Hybrid attention (§2.3)": shared K=V MQA (one KV head
# read as key and value), partial RoPE and the -i output rotation (eq. 26),
# per-head learnable sink (eq. 27), the sliding-window K=V branch concatenated
# with the compressor output before core attention; "Attention mask layout".
# --------------------------------------------------------------------------
def attend_row(q_rot, keys, sink, scale, dv):
    """Softmax attention of H query heads over one shared K=V key set plus a sink.

    logits l[h,j] = scale * q[h] . k_j ; value v_j = k_j[:dv] (K=V);
    o[h] = sum_j e^{l[h,j]} v_j / (e^{sink[h]} + sum_j e^{l[h,j]})   (reading R5).
    """
    q_rot = _f64(q_rot)
    keys = _f64(keys)
    sink = _f64(sink)
    H = q_rot.shape[0]
    if keys.shape[0] == 0:
        return np.zeros((H, dv))
    logits = scale * (q_rot @ keys.T)  # [H, Nk]
    mx = np.maximum(logits.max(axis=1), sink)
    e = np.exp(logits - mx[:, None])
    denom = e.sum(axis=1) + np.exp(sink - mx)
    return (e @ keys[:, :dv]) / denom[:, None]


def sparse_mqa_attention(q, kv_win, pool, idx, sink, qpos, q_index, *, n_win, m,
                         scale, dv, R, theta, rope_q, rotate_out, win_ring=0,
                         P_cap=None, rows=None):
    """Per query: keys = window rows (t-n_win, t] + pool entries idx[b,s] (!= -1).

    q [B,Sq,H,D]; kv_win: window rows already rotated, [B,S,D] indexed by cache
    index, or a ring [B,win_ring,D] (token j in slot j % win_ring); pool [B,P,D]
    already rotated; idx [B,Sq,K] or None (= every visible entry, HCA);
    sink [H]; qpos [B,Sq] RoPE positions; q_index [B,Sq] cache indices.
    rope_q: rotate q at qpos first.  rotate_out: rotate the output rope slice by
    -qpos (eq. 26).  Returns out [B,Sq,H,dv] (rows not computed stay 0).
    """
    B, Sq, H, D = q.shape
    P = pool.shape[1] if P_cap is None else P_cap
    out = np.zeros((B, Sq, H, dv))
    if rows is None:
        rows = [(b, s) for b in range(B) for s in range(Sq)]
    for b, s in rows:
        t = int(q_index[b, s])
        q_t = rope_rotate(q[b, s], qpos[b, s], R, theta) if rope_q else _f64(q[b, s])
        win = window_tokens(t, n_win)
        slots = [j % win_ring for j in win] if win_ring else win
        vis = visible_entries(t, m, P)
        if idx is None:
            sel = list(range(vis))
        else:
            sel = [int(w) for w in idx[b, s] if w >= 0]
            assert all(w < vis for w in sel), "selected pool entry is not visible"
            assert len(set(sel)) == len(sel), "pool entry selected twice"
        keys = np.concatenate([_f64(kv_win[b, slots]).reshape(len(slots), D),
                               _f64(pool[b, sel]).reshape(len(sel), D)], axis=0)
        o = attend_row(q_t, keys, sink, scale, dv)
        if rotate_out:
            assert dv == D, "output rotation needs the rope slice in the value"
            o = rope_rotate(o, qpos[b, s], R, theta, sign=-1.0)
        out[b, s] = o
    return out


# --------------------------------------------------------------------------
# Layers (prefill): [V4] CSA = compressor + indexer + core attention;
# HCA = compressor + core attention over every visible entry (no indexer).
# --------------------------------------------------------------------------
def csa_layer(q, kv, z, bias, qI, wI, kI, zI, biasI, sink, pos, *, m, overlap,
              n_win, topk, scale, dv, R, theta, rotate_out, rows=None, store=None):
    """Prefill CSA layer (Sq == S, query s sits at cache index s).

    ``store`` rounds the pools and the rotated window rows to the dtype a cache keeps
    them in before they are read again (see ``store_as``).
    """
    B, S = kv.shape[0], kv.shape[1]
    pool = store_as(compress(kv, z, bias, pos, m=m, overlap=overlap, apply_rope=True, R=R,
                             theta=theta), store)
    poolI = store_as(compress(kI, zI, biasI, pos, m=m, overlap=overlap, apply_rope=False), store)
    kv_rot = store_as(rope_rotate(kv, pos, R, theta), store)
    q_index = np.tile(np.arange(S), (B, 1))
    idx = indexer_topk(qI, wI, poolI, q_index, m=m, topk=topk, rows=rows)
    out = sparse_mqa_attention(q, kv_rot, pool, idx, sink, pos, q_index, n_win=n_win, m=m,
                               scale=scale, dv=dv, R=R, theta=theta, rope_q=True,
                               rotate_out=rotate_out, rows=rows)
    return {"pool": pool, "poolI": poolI, "kv_rot": kv_rot, "idx": idx, "out": out}


def hca_layer(q, kv, z, bias, sink, pos, *, m, n_win, scale, dv, R, theta, rotate_out,
              rows=None, store=None):
    """Prefill HCA layer: non-overlapping pool, every visible entry attended."""
    B, S = kv.shape[0], kv.shape[1]
    pool = store_as(compress(kv, z, bias, pos, m=m, overlap=False, apply_rope=True, R=R,
                             theta=theta), store)
    kv_rot = store_as(rope_rotate(kv, pos, R, theta), store)
    q_index = np.tile(np.arange(S), (B, 1))
    out = sparse_mqa_attention(q, kv_rot, pool, None, sink, pos, q_index, n_win=n_win, m=m,
                               scale=scale, dv=dv, R=R, theta=theta, rope_q=True,
                               rotate_out=rotate_out, rows=rows)
    return {"pool": pool, "kv_rot": kv_rot, "out": out}


def sliding_layer(q, kv, sink, pos, *, n_win, scale, dv, R, theta, rotate_out, rows=None, store=None):
    """Prefill sliding-window layer ([V4] layer types, `sliding_attention`): no compressor
    and no indexer; the K=V rows rotated at their positions, then attention over the
    window (t - n_win, t] alone."""
    B, S, D = kv.shape
    kv_rot = store_as(rope_rotate(kv, pos, R, theta), store)
    q_index = np.tile(np.arange(S), (B, 1))
    out = sparse_mqa_attention(q, kv_rot, np.zeros((B, 0, D)), None, sink, pos, q_index, n_win=n_win, m=1,
                               scale=scale, dv=dv, R=R, theta=theta, rope_q=True,
                               rotate_out=rotate_out, P_cap=0, rows=rows)
    return {"kv_rot": kv_rot, "out": out}


# --------------------------------------------------------------------------
# Grouped output projection  [V4] "Hybrid attention (§2.3)", grouped low-rank output
# projection (o_a_proj, a grouped linear, then o_b_proj; o_groups, o_lora_rank).
# --------------------------------------------------------------------------
def grouped_out_proj(o, wa, wb):
    """o [T,H,dv] attention outputs; wa [g, d_g, (H/g)*dv] one o_a_proj weight per head group;
    wb [hidden, g*d_g] the o_b_proj weight.  Returns y [T, hidden] (no biases).

    Reading R14: group i holds the contiguous heads [i*H/g, (i+1)*H/g); its heads' outputs,
    concatenated in head order, are projected by its own weight to d_g channels; the g
    results, concatenated in group order, are projected to hidden_size.
    """
    T, H, dv = o.shape
    g = wa.shape[0]
    assert H % g == 0 and wa.shape[2] == (H // g) * dv and wb.shape[1] == g * wa.shape[1]
    hg = H // g
    o = _f64(o)
    u = np.concatenate([o[:, i * hg:(i + 1) * hg, :].reshape(T, hg * dv) @ _f64(wa[i]).T for i in range(g)], axis=1)
    return u @ _f64(wb).T


# --------------------------------------------------------------------------
# Decode cache  [V4] "Cache layers": the CSA / HCA cache keeps the sliding window of
# K=V rows and the compressor's buffer of the tokens of the open window(s) (for CSA the
# previous block too: the overlap state); an entry is emitted every m tokens.  The
# indexer keys keep a buffer and a pool of their own.
# --------------------------------------------------------------------------
def new_decode_cache(c, *, m, overlap, P_cap, win_ring=0):
    """Empty cache of one stream of one sequence: a buffer of the last Lw = 2m (overlap)
    or m raw token rows with their logits and positions, an optional window ring and the
    pool."""
    lw = 2 * m if overlap else m
    return {"raw": np.zeros((lw, c)), "z": np.zeros((lw, c)), "pos": np.zeros(lw, dtype=np.int64),
            "win": np.zeros((win_ring, c)) if win_ring else None, "pool": np.zeros((P_cap, c))}


def decode_append(cache, x_t, z_t, pos_t, t, *, m, overlap, bias, apply_rope, R=0, theta=160000.0):
    """Append token t (cache index) of one sequence: row x_t [c] (not rotated), logits z_t
    [c] or None, position pos_t.  Tokens must arrive in order t = 0, 1, 2, ...

    The buffer holds token j in slot j % Lw; the window ring holds token j rotated at its
    position in slot j % win_ring.  When t closes a block ((t+1) % m == 0), entry
    w = (t+1)/m - 1 is pooled from the buffered tokens of its window (readings R1-R3: the
    softmax over z + the per-slot bias, rotated at the position of the first token of its
    own block) and written to the pool if w < P_cap.
    """
    lw = cache["raw"].shape[0]
    c = cache["raw"].shape[1]
    cache["raw"][t % lw] = _f64(x_t)
    cache["z"][t % lw] = 0.0 if z_t is None else _f64(z_t)
    cache["pos"][t % lw] = pos_t
    if cache["win"] is not None:
        row = rope_rotate(_f64(x_t), pos_t, R, theta) if apply_rope else _f64(x_t)
        cache["win"][t % cache["win"].shape[0]] = row
    if (t + 1) % m != 0:
        return
    w = (t + 1) // m - 1
    if w >= cache["pool"].shape[0]:
        return
    lo = (w - 1) * m if overlap else w * m
    tokens = [j for j in range(max(lo, 0), t + 1)]
    logit = np.zeros((len(tokens), c))
    for k, j in enumerate(tokens):
        logit[k] = cache["z"][j % lw]
        if bias is not None:
            logit[k] = logit[k] + _f64(bias)[j - lo]
    mx = logit.max(axis=0)
    e = np.exp(logit - mx)
    alpha = e / e.sum(axis=0)
    entry = sum(alpha[k] * cache["raw"][j % lw] for k, j in enumerate(tokens))
    if apply_rope:
        entry = rope_rotate(entry, cache["pos"][(w * m) % lw], R, theta)
    cache["pool"][w] = entry
