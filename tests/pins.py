"""Checks that pin the CPU oracle to things other than itself.

Each ``check_*`` raises AssertionError when the oracle disagrees with the pin:
a library routine computing the same definition (torch fp64
scaled_dot_product_attention, torch.sort, torch.logsumexp), a closed form or
invariant, or a hand-enumerated case from ``tests/golden``.  The pin tests call
them on the oracle as written; the mutation tests call them on deliberately
broken copies and expect them to fail.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

from oracle import csa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _sdpa(q, k, v, mask=None, scale=None, is_causal=False):
    """torch fp64 attention: q [H, m, D], k/v [H, n, D], mask [H or 1, m, n] bool."""
    return F.scaled_dot_product_attention(
        torch.tensor(np.array(q), dtype=torch.float64)[None], torch.tensor(np.array(k), dtype=torch.float64)[None],
        torch.tensor(np.array(v), dtype=torch.float64)[None],
        attn_mask=None if mask is None else torch.tensor(np.array(mask))[None],
        scale=scale, is_causal=is_causal)[0].numpy()


# ---------------------------------------------------------------- attention

def check_attention_vs_sdpa(seed=0, G=4, D=32, T=512, L=32, n_sel=5):
    """Sparse attention over a chunk set == fp64 SDPA with a mask that keeps
    exactly the tokens of those chunks; lse == logsumexp of the masked logits."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((G, D))
    K = rng.standard_normal((T, D))
    V = rng.standard_normal((T, D))
    C = T // L
    chunks = sorted(rng.choice(C, size=n_sel, replace=False).tolist())
    scale = 1.0 / math.sqrt(D)
    o, lse = O.decode_unit(q, K, V, chunks, L, scale)
    keep = np.zeros(T, dtype=bool)
    for c in chunks:
        keep[c * L:(c + 1) * L] = True
    mask = np.broadcast_to(keep, (G, 1, T))
    ref = _sdpa(q[:, None, :], np.broadcast_to(K, (G, T, D)), np.broadcast_to(V, (G, T, D)),
                mask=mask, scale=scale)[:, 0]
    assert np.allclose(o, ref, rtol=0, atol=1e-12), np.abs(o - ref).max()
    logits = torch.as_tensor(q @ K.T * scale)
    logits[:, ~torch.as_tensor(keep)] = -math.inf
    ref_lse = torch.logsumexp(logits, dim=1).numpy()
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def check_dense_special_case(seed=1, G=2, D=16, T=256, L=32):
    """Selecting every chunk (k_free covers the pool) reduces to dense
    attention: fp64 SDPA with no mask."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((G, D))
    K = rng.standard_normal((T, D))
    V = rng.standard_normal((T, D))
    C = T // L
    summ = O.chunk_summaries(K, L)
    s = O.score_chunks(q[None, None], summ[None, None], 1)[0, 0, 0]
    chunks, _ = O.select_topk(s, C, 1, 1)
    assert chunks == list(range(C))
    o, _ = O.decode_unit(q, K, V, chunks, L, 0.25)
    ref = _sdpa(q[:, None, :], np.broadcast_to(K, (G, T, D)), np.broadcast_to(V, (G, T, D)),
                scale=0.25)[:, 0]
    assert np.allclose(o, ref, rtol=0, atol=1e-12)


def check_empty_attention():
    """An empty token set gives o = 0 and lse = -inf (no NaN)."""
    o, lse = O.attend(np.ones((2, 4)), np.ones((8, 4)), np.ones((8, 4)), np.zeros(0, dtype=int), 1.0)
    assert np.all(o == 0) and np.all(lse == -math.inf)


def check_hybrid_golden():
    """Hybrid context in both gist scopes ("selected": gist and raw KV of the
    chosen chunks; "all": every chunk's gist plus the raw KV of the chosen
    ones): the hand-worked cases of tests/golden/hybrid_cases.json."""
    g = _golden("hybrid_cases.json")
    q, K, V = (np.array(g[k], dtype=np.float64) for k in ("q", "K", "V"))
    Kg, Vg = np.array(g["Kg"], dtype=np.float64), np.array(g["Vg"], dtype=np.float64)
    for scope in ("all", "selected"):
        for c in g["cases_" + scope]:
            o, lse = O.hybrid_unit(q, K, V, Kg, Vg, c["chunks"], g["L"], g["scale"], scope)
            want_lse = np.array([float(x) for x in c["lse"]])
            assert np.allclose(o, np.array(c["o"]), rtol=0, atol=1e-12), (scope, c["chunks"], o)
            assert np.array_equal(np.isinf(lse), np.isinf(want_lse)), (scope, c["chunks"], lse)
            fin = np.isfinite(want_lse)
            assert np.allclose(lse[fin], want_lse[fin], rtol=0, atol=1e-12), (scope, c["chunks"], lse)


def check_hybrid_vs_sdpa(seed=16, G=4, D=16, T=256, L=32):
    """Hybrid context == fp64 SDPA over the raw cache with the C gist rows
    appended, masked to keep the selected chunks' raw tokens and the gist
    rows of the scope (the selected chunks' own, or every chunk's); lse ==
    logsumexp of the same masked logits.  Chunk sets from empty to all
    chunks (an empty set in the "selected" scope has nothing to attend)."""
    rng = np.random.default_rng(seed)
    C = T // L
    for scope in ("all", "selected"):
        for n_sel in (0, 1, 3, C):
            q = rng.standard_normal((G, D))
            K, V = rng.standard_normal((T, D)), rng.standard_normal((T, D))
            Kg, Vg = rng.standard_normal((C, D)), rng.standard_normal((C, D))
            chunks = sorted(rng.choice(C, size=n_sel, replace=False).tolist())
            scale = 1.0 / math.sqrt(D)
            o, lse = O.hybrid_unit(q, K, V, Kg, Vg, chunks, L, scale, scope)
            Ke, Ve = np.concatenate([K, Kg]), np.concatenate([V, Vg])
            keep = np.zeros(T + C, dtype=bool)
            for c in chunks:
                keep[c * L:(c + 1) * L] = True
                keep[T + c] = scope == "selected"
            if scope == "all":
                keep[T:] = True
            if not keep.any():
                assert np.all(o == 0) and np.all(lse == -math.inf), (scope, o, lse)
                continue
            mask = np.broadcast_to(keep, (G, 1, T + C))
            ref = _sdpa(q[:, None, :], np.broadcast_to(Ke, (G, T + C, D)),
                        np.broadcast_to(Ve, (G, T + C, D)), mask=mask, scale=scale)[:, 0]
            assert np.allclose(o, ref, rtol=0, atol=1e-12), (scope, np.abs(o - ref).max())
            logits = torch.as_tensor(q @ Ke.T * scale)
            logits[:, ~torch.as_tensor(keep)] = -math.inf
            assert np.allclose(lse, torch.logsumexp(logits, dim=1).numpy(), rtol=0, atol=1e-12)


def check_pipeline_topp_scale_under_projection():
    """The decode step's top-p branch softmaxes the (projected) chunk scores
    with the attention scale 1/sqrt(D) of the head dimension D, not
    1/sqrt(R) of the projection rank and not the caller's attention scale.
    Hand case: D = 4, R = 2, P = the first two unit vectors, q = e0, four
    chunks of two identical keys, chunk 1's keys e0 * 2 ln 3, the others 0.
    Scores (0, 2 ln 3, 0, 0).  With 1/sqrt(D) = 1/2 the weights are
    (1, 3, 1, 1): chunk 1 holds 1/2 < p = 0.6, and chunk 0 (ties to the lower
    index) brings the prefix to 2/3, so the set is {0, 1}.  With 1/sqrt(R)
    the weight of chunk 1 is 3^sqrt(2) (mass 0.61 >= 0.6) and with scale 1
    it is 9 (mass 3/4): both would give {1}."""
    from oracle import pipeline as OP
    D, L, C = 4, 2, 4
    K = np.zeros((1, 1, C * L, D))
    K[0, 0, 1 * L:2 * L, 0] = 2.0 * math.log(3.0)
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 1.0
    P = np.zeros((D, 2))
    P[0, 0] = P[1, 1] = 1.0
    res = OP.decode_step(q, K, np.zeros_like(K), L=L, scale=1.0, select="topp", n_sink=0,
                         n_local=0, proj=P, p=0.6, budget=C, with_attention=False)
    assert res["sets"][(0, 0)] == [0, 1], res["sets"]
    assert res["n_p"][(0, 0)] == 2, res["n_p"]


def check_pipeline_rope_branch():
    """The decode step's RoPE branch: the query sits at position T - 1 (the
    context's last token), and with a bf16 cache the rotated query and keys
    are held in bf16.  Hand case: D = 2 (one pair turning by pos radians),
    L = 1, T = 2, q = e0, keys e0 and e0, values e0 and e1, scale 1.
    fp64 inputs: the rotated query at position 1 meets k0 (position 0) with
    cos(1 - 0) and k1 (position 1) with cos 0 = 1, so the weight of v0 is
    1 / (1 + e^(1 - cos 1)); a query at position T = 2 would give
    1 / (1 + e^(cos 1 - cos 2)).  bf16 inputs: cos 1 = 0.5403 and
    sin 1 = 0.8415 lie in [0.5, 1), where bf16 steps by 2^-8, so they are
    held as 138/256 and 215/256; the logits become 138/256 and
    (138^2 + 215^2)/256^2 and the weight of v0 is
    1 / (1 + e^((138^2 + 215^2)/65536 - 138/256))."""
    from oracle import pipeline as OP
    for dtype in (torch.float64, torch.bfloat16):
        q = torch.tensor([[[1.0, 0.0]]], dtype=dtype)
        K = torch.tensor([[[[1.0, 0.0], [1.0, 0.0]]]], dtype=dtype)
        V = torch.tensor([[[[1.0, 0.0], [0.0, 1.0]]]], dtype=dtype)
        res = OP.decode_step(q, K, V, L=1, scale=1.0, select="topk", n_sink=1, n_local=1,
                             k_free=0, rope_theta=10000.0)
        assert res["sets"][(0, 0)] == [0, 1]
        if dtype == torch.float64:
            w0 = 1.0 / (1.0 + math.exp(1.0 - math.cos(1.0)))
        else:
            w0 = 1.0 / (1.0 + math.exp((138 ** 2 + 215 ** 2) / 65536.0 - 138 / 256.0))
        o = res["o"][(0, 0)]
        assert np.allclose(o, [[w0, 1.0 - w0]], rtol=0, atol=1e-12), (dtype, o, w0)


def check_rope_closed_forms(seed=18):
    """RoPE: hand-worked pairs (D = 2: a rotation by pos radians; D = 4: the
    pairing and the frequencies);
    position 0 is the identity; norms are kept; and the textbook relative
    property q(m).k(n) = q(m - n).k(0) for every pair of positions."""
    x = np.array([[1.0, 0.0], [0.0, 2.0]])
    y = O.rope(x, [math.pi / 2, math.pi / 6], 10000.0)
    assert np.allclose(y, [[0.0, 1.0], [-1.0, math.sqrt(3.0)]], atol=1e-15), y
    # D = 4, theta = 100: pairs (0, 2) at frequency 1 and (1, 3) at 100^(-1/2)
    # = 0.1 (rotate-half pairing, frequency theta^(-2i/D)); position pi/2
    y = O.rope(np.eye(4)[:2], [math.pi / 2, math.pi / 2], 100.0)
    c, s_ = math.cos(math.pi / 20), math.sin(math.pi / 20)
    assert np.allclose(y, [[0.0, 0.0, 1.0, 0.0], [0.0, c, 0.0, s_]], atol=1e-15), y
    rng = np.random.default_rng(seed)
    D = 16
    q, k = rng.standard_normal((5, D)), rng.standard_normal((5, D))
    assert np.array_equal(O.rope(q, np.zeros(5), 500.0), q)
    m = np.array([0, 3, 17, 1000, 131071], dtype=np.float64)
    assert np.allclose(np.linalg.norm(O.rope(q, m, 500.0), axis=1), np.linalg.norm(q, axis=1),
                       rtol=1e-12)
    for mi in m:
        for ni in (0.0, 5.0, 999.0):
            lhs = O.rope(q, np.full(5, mi), 500.0) @ O.rope(k, np.full(5, ni), 500.0).T
            rhs = O.rope(q, np.full(5, mi - ni), 500.0) @ k.T
            assert np.allclose(lhs, rhs, rtol=0, atol=1e-9), (mi, ni)


def check_token_sparse_golden():
    """Token importance and the coverage budget on the hand-worked cases of
    tests/golden/token_sparse_cases.json."""
    g = _golden("token_sparse_cases.json")
    im = g["importance"]
    got = O.token_importance(np.array(im["Q_obs"]), np.array(im["K"]), np.array(im["obs_pos"]),
                             im["scale"])
    assert np.allclose(got, im["expected"], rtol=0, atol=1e-12), got
    for tau, k in g["budget"]["cases"]:
        assert O.coverage_budget(g["budget"]["mass"], tau) == k, (tau, k)


def check_token_sparse_invariants(seed=22, trials=30):
    """Importance: every query row spends a total weight of 1; keys after a
    row's position get none from it.  Budget: equals the smallest m whose m
    most important tokens hold >= 1 - tau of the mass (the same cut counted
    from the top), on cases without near-ties.  Token choice: torch.sort on
    (score desc, index asc)."""
    rng = np.random.default_rng(seed)
    S, D, r = 40, 8, 6
    q, k = rng.standard_normal((r, D)), rng.standard_normal((S, D))
    pos = np.array([39, 38, 30, 20, 5, 0])
    im = O.token_importance(q, k, pos, 0.5)
    assert abs(im.sum() - r) < 1e-9
    assert im[39] > 0 and abs(O.token_importance(q[4:5], k, pos[4:5], 0.5)[6:].sum()) == 0.0
    for _ in range(trials):
        n = int(rng.integers(2, 60))
        m = rng.random(n) ** 3
        m /= m.sum()
        tau = float(rng.random() * 0.5)
        srt = np.sort(m)[::-1]
        cum = np.cumsum(srt)
        if np.min(np.abs(cum - (1 - tau))) < 1e-9:
            continue
        m_top = int(np.argmax(cum >= 1 - tau - 1e-15)) + 1
        assert O.coverage_budget(m, tau) == m_top, (n, tau)
        kk = int(rng.integers(0, n + 1))
        sc = np.round(rng.standard_normal(n), 1)  # ties on purpose
        ref = sorted(torch.sort(torch.tensor(-sc * 1000.0 + np.arange(n) * 1e-3)).indices[:kk].tolist())
        assert O.select_tokens(sc, kk) == ref


def check_token_sparse_vs_sdpa(seed=23, S=96, G=2, D=16):
    """Compress, dense causal attention, decompress == fp64 SDPA over the
    whole sequence with a mask keeping, for a selected query row, the
    selected keys at or before it; rows not selected are 0."""
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((S, G, D))
    K, V = rng.standard_normal((S, D)), rng.standard_normal((S, D))
    sel = sorted(rng.choice(S, size=37, replace=False).tolist())
    out = O.token_sparse_head(Q, K, V, sel, 0.25)
    keep = np.zeros(S, dtype=bool)
    keep[sel] = True
    mask = keep[:, None] & keep[None, :] & (np.arange(S)[None, :] <= np.arange(S)[:, None])
    mask[~keep, 0] = True  # rows left out get a dummy key; compared as zeros below
    for g in range(G):
        ref = _sdpa(Q[None, :, g], K[None], V[None], mask=mask[None], scale=0.25)[0]
        assert np.allclose(out[keep, g], ref[keep], rtol=0, atol=1e-12)
        assert np.all(out[~keep, g] == 0)


# ---------------------------------------------------------------- summaries / scores

def check_summary_closed_form():
    """Keys that are constant within a chunk (row value = chunk id + column id)
    have exactly that constant as summary; the projected summary equals the
    mean of the projected keys (linearity)."""
    L, C, D = 4, 5, 3
    K = np.zeros((C * L, D))
    for c in range(C):
        K[c * L:(c + 1) * L] = c + np.arange(D)
    s = O.chunk_summaries(K, L)
    assert np.array_equal(s, np.arange(C)[:, None] + np.arange(D)[None, :])
    rng = np.random.default_rng(3)
    K = rng.standard_normal((8 * 16, 12))
    P = rng.standard_normal((12, 4)) / 4
    a = O.chunk_summaries(K, 16, P)
    b = (K @ P).reshape(8, 16, 4).mean(axis=1)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def check_score_hand_case():
    """s = q^T k_summary summed over the query heads of the KV head, on a case
    worked by hand: heads q0 = (1, 2), q1 = (3, -1); summaries (1, 0), (0, 1),
    (2, 2).  Group sum (4, 1): scores 4, 1, 10."""
    q = np.array([[[[1.0, 2.0], [3.0, -1.0]]]])  # [B=1, Nq=1, Hq=2, D=2]
    summ = np.array([[[[1.0, 0.0], [0.0, 1.0], [2.0, 2.0]]]])  # [1, Hkv=1, C=3, 2]
    s = O.score_chunks(q, summ, 1)
    assert np.array_equal(s[0, 0, 0], [4.0, 1.0, 10.0])
    # two KV heads each with one query head: no mixing across groups
    q2 = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    summ2 = np.array([[[[5.0, 7.0]], [[5.0, 7.0]]]])  # [1, 2, 1, 2]
    s2 = O.score_chunks(q2, summ2, 2)
    assert s2[0, 0, 0, 0] == 5.0 and s2[0, 1, 0, 0] == 7.0


def check_projection_closed_form(seed=4):
    """(P^T q) . (P^T kbar) == q^T (P P^T) kbar, computed two ways."""
    rng = np.random.default_rng(seed)
    D, R, C, G = 24, 6, 7, 3
    q = rng.standard_normal((1, 1, G, D))
    kbar = rng.standard_normal((C, D))
    P = rng.standard_normal((D, R)) / 4
    s = O.score_chunks(q, (kbar @ P)[None, None], 1, P)[0, 0, 0]
    ref = (q[0, 0].sum(axis=0) @ P @ P.T) @ kbar.T
    assert np.allclose(s, ref, rtol=0, atol=1e-12)


def check_tile_mean():
    """Tile mean of rows that are constant within the tile is that row; means
    of a linear ramp are the ramp's midpoints."""
    B, S, Hq, D, m = 1, 12, 2, 3, 4
    Q = np.zeros((B, S, Hq, D))
    for s_ in range(S):
        Q[0, s_] = s_
    tm = O.tile_mean_q(Q, m)
    assert np.array_equal(tm[0, :, 0, 0], [1.5, 5.5, 9.5])


# ---------------------------------------------------------------- selection

def check_topk_golden():
    for c in _golden("topk_cases.json")["cases"]:
        got, _ = O.select_topk(np.array(c["scores"], dtype=np.float64), c["k_free"],
                               c["n_sink"], c["n_local"], c["n_valid"])
        assert got == c["expect"], (c["why"], got)


def check_topk_vs_torch_sort(seed=5, C=64, trials=20):
    """Library pin: the free part of the set is the first k_free of a stable
    descending torch.sort over the non-forced chunks (stable sort keeps equal
    scores in ascending index order)."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        s = rng.integers(-4, 5, size=C).astype(np.float64)  # many exact ties
        n_sink, n_local = int(rng.integers(0, 3)), int(rng.integers(0, 3))
        k_free = int(rng.integers(0, C))
        got, _ = O.select_topk(s, k_free, n_sink, n_local)
        forced = set(range(n_sink)) | set(range(C - n_local, C))
        pool = torch.tensor([c for c in range(C) if c not in forced], dtype=torch.long)
        order = torch.sort(torch.as_tensor(s)[pool], descending=True, stable=True).indices
        ref = sorted(forced | set(pool[order[:k_free]].tolist()))
        assert got == ref


def check_topk_invariants(seed=6, C=40, trials=20):
    """Forced chunks present; size = |F| + min(k_free, pool); every chosen
    pool chunk scores >= every unchosen pool chunk; output ascending."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        s = rng.standard_normal(C)
        v = int(rng.integers(1, C + 1))
        k_free = int(rng.integers(0, C))
        got, _ = O.select_topk(s, k_free, 1, 1, v)
        F_ = {0, v - 1}
        assert F_ <= set(got) and got == sorted(got) and all(c < v for c in got)
        pool = [c for c in range(v) if c not in F_]
        chosen = [c for c in got if c not in F_]
        assert len(chosen) == min(k_free, len(pool))
        rest = [c for c in pool if c not in chosen]
        if chosen and rest:
            assert min(s[chosen]) >= max(s[rest])


def check_topk_union_golden():
    for c in _golden("topk_union_cases.json")["cases"]:
        got, _ = O.select_topk_union(np.array(c["scores"], dtype=np.float64), c["k_free"],
                                     c["n_sink"], c["n_local"])
        assert got == c["expect"], (c["why"], got)


def check_topk_union_brute_force(seed=14, G=3, C=12, trials=40):
    """Brute force on tiny inputs with many exact ties: a non-forced chunk is
    in the union iff, for some head, fewer than k_free non-forced chunks beat
    it (higher score, or equal score and lower index).  A single head gives
    the unit top-k."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        s = rng.integers(-2, 3, size=(G, C)).astype(np.float64)
        n_sink, n_local = int(rng.integers(0, 3)), int(rng.integers(0, 3))
        k_free = int(rng.integers(0, C))
        got, _ = O.select_topk_union(s, k_free, n_sink, n_local)
        forced = set(range(min(n_sink, C))) | set(range(max(C - n_local, 0), C))
        pool = [c for c in range(C) if c not in forced]
        ref = set(forced)
        for c in pool:
            for g in range(G):
                beaten_by = sum(1 for d in pool if s[g, d] > s[g, c] or (s[g, d] == s[g, c] and d < c))
                if beaten_by < k_free:
                    ref.add(c)
                    break
        assert got == sorted(ref), (got, sorted(ref))
        one, _ = O.select_topk_union(s[:1], k_free, n_sink, n_local)
        flat, _ = O.select_topk(s[0], k_free, n_sink, n_local)
        assert one == flat


def check_per_head_scores(seed=15):
    """Per-head scores: a hand case, and their sum over the heads equals the
    group-summed score of score_chunks (pinned by its own hand case)."""
    q = np.array([[1.0, 0.0], [0.0, 2.0]])
    summ = np.array([[3.0, 4.0], [1.0, -1.0], [0.5, 0.0]])
    assert np.array_equal(O.score_chunks_per_head(q, summ), [[3.0, 1.0, 0.5], [8.0, -2.0, 0.0]])
    rng = np.random.default_rng(seed)
    G, D, C, R = 4, 16, 9, 8
    q = rng.standard_normal((G, D))
    summ = rng.standard_normal((C, R))
    P = rng.standard_normal((D, R))
    per = O.score_chunks_per_head(q, summ, P)
    grp = O.score_chunks(q[None, None], summ[None, None], 1, P)[0, 0, 0]
    assert np.allclose(per.sum(axis=0), grp, rtol=0, atol=1e-12)


def check_topp_golden():
    for c in _golden("topp_cases.json")["cases"]:
        got, n_p, _ = O.select_topp(np.array(c["scores"], dtype=np.float64), c["logit_scale"],
                                    c["p"], c["budget"], c["n_sink"], c["n_local"])
        assert got == c["expect"] and n_p == c["n_p"], (c["why"], got, n_p)


def check_topp_invariants(seed=7, C=50, trials=30):
    """cum(n_p - 1) < p <= cum(n_p) on the mass sorted by numpy (library);
    forced chunks present; |set| <= budget + |F|; when n_p <= budget the free
    part is exactly the n_p largest masses."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        s = rng.standard_normal(C) * rng.uniform(0.5, 8)
        p = float(rng.uniform(0.05, 0.99))
        budget = int(rng.integers(1, C))
        scale = float(rng.uniform(0.1, 2))
        got, n_p, _ = O.select_topp(s, scale, p, budget, 1, 2)
        pi = np.exp(s * scale - (s * scale).max())
        pi /= pi.sum()
        cum = np.cumsum(np.sort(pi)[::-1])
        assert cum[n_p - 1] >= p and (n_p == 1 or cum[n_p - 2] < p)
        F_ = {0, C - 2, C - 1}
        assert F_ <= set(got) and len(got) <= budget + len(F_)
        if n_p <= budget:
            top = set(np.argsort(-pi, kind="stable")[:n_p].tolist())
            assert set(got) == top | F_


def check_hier_golden():
    for c in _golden("hier_cases.json")["cases"]:
        summ = np.array(c["summ"], dtype=np.float64)[:, None]
        meta = O.meta_summaries(summ, c["Gm"])
        got, _, _ = O.select_hier(np.array(c["q"]), meta, summ, c["Gm"], c["top_meta"],
                                  c["k_free"], c["n_sink"], c["n_local"])
        assert got == c["expect"], (c["why"], got)


def check_hier_all_metas_is_flat(seed=8, trials=10):
    """Keeping every meta-chunk reduces the hierarchy to flat top-k over all
    chunks with the same forced set and k_free."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        G, D, Gm, M = 4, 16, 8, 12
        C = Gm * M
        q = rng.standard_normal((G, D))
        summ = rng.standard_normal((C, D))
        meta = O.meta_summaries(summ, Gm)
        k_free = int(rng.integers(1, 30))
        got, _, _ = O.select_hier(q, meta, summ, Gm, M, k_free, 1, 2)
        s = O.score_chunks(q[None, None], summ[None, None], 1)[0, 0, 0]
        flat, _ = O.select_topk(s, k_free, 1, 2)
        assert got == flat


def check_meta_linearity(seed=9):
    """A meta-summary (mean of Gm chunk means) equals the plain mean of all
    Gm * L raw keys under it."""
    rng = np.random.default_rng(seed)
    L, Gm, M, D = 8, 4, 3, 5
    K = rng.standard_normal((L * Gm * M, D))
    meta = O.meta_summaries(O.chunk_summaries(K, L), Gm)
    ref = K.reshape(M, Gm * L, D).mean(axis=1)
    assert np.allclose(meta, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- split-K and merge

def check_merge_closed_form(seed=10, trials=10):
    """Merging partials of any partition of a token set equals one-pass
    attention over the set; an empty (-inf) split contributes nothing; one
    partial merges to itself."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        G, D, n = 3, 8, int(rng.integers(2, 60))
        q = rng.standard_normal((G, D)) * 2
        K = rng.standard_normal((n, D))
        V = rng.standard_normal((n, D))
        tok = np.arange(n)
        o_ref, lse_ref = O.attend(q, K, V, tok, 0.7)
        cuts = sorted(rng.choice(np.arange(1, n), size=int(rng.integers(1, min(n, 6))),
                             replace=False).tolist())
        parts = np.split(tok, cuts)
        op, lp = [], []
        for pt in parts:
            o, l = O.attend(q, K, V, pt, 0.7)
            op.append(o)
            lp.append(l)
        op.append(np.full((G, D), 123.0))  # an empty split: o must not be read
        lp.append(np.full(G, -math.inf))
        o_part = np.stack(op, axis=1)
        lse_part = np.stack(lp, axis=1)
        om, lm = O.lse_merge(o_part, lse_part)
        assert np.allclose(om, o_ref, rtol=0, atol=1e-12)
        assert np.allclose(lm, lse_ref, rtol=0, atol=1e-12)
        o1, l1 = O.lse_merge(o_ref[:, None], lse_ref[:, None])
        assert np.allclose(o1, o_ref, rtol=0, atol=1e-14) and np.allclose(l1, lse_ref, atol=1e-14)


def check_partition(seed=11, trials=20):
    """The split-K layout covers each unit's list exactly once, in order, with
    pieces whose sizes differ by at most one across the whole job."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        n = rng.integers(0, 40, size=int(rng.integers(1, 9))).tolist()
        P = int(rng.integers(1, 50))
        spl = O.decode_partition(n, P)
        for u, s in enumerate(spl):
            pos = 0
            for (a, b) in s:
                assert a == pos and b > a
                pos = b
            assert pos == n[u]
        N = sum(n)
        sizes = [((c + 1) * N) // P - (c * N) // P for c in range(P)]
        assert max(sizes) - min(sizes) <= 1
        assert sum(len(s) for s in spl) <= P + len(n) - 1
    # hand-worked: lists of 5 and 3 chunks, 3 pieces: cuts at 0, 2, 5, 8
    assert O.decode_partition([5, 3], 3) == [[(0, 2), (2, 5)], [(0, 3)]]
    # lists of 4 and 4, 3 pieces: piece [2, 5) straddles the two units
    assert O.decode_partition([4, 4], 3) == [[(0, 2), (2, 4)], [(0, 1), (1, 4)]]
    # more pieces than chunks: empty pieces produce no split
    assert O.decode_partition([2, 0, 1], 5) == [[(0, 1), (1, 2)], [], [(0, 1)]]


# ---------------------------------------------------------------- prefill

def check_prefill_dense_causal(seed=12, S=256, L=32, D=16, G=2):
    """When every visible chunk is selected the block-sparse prefill is plain
    causal attention: fp64 SDPA with is_causal=True."""
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((G, S, D))
    K = rng.standard_normal((S, D))
    V = rng.standard_normal((S, D))
    ref = _sdpa(Q, np.broadcast_to(K, (G, S, D)), np.broadcast_to(V, (G, S, D)),
                scale=0.3, is_causal=True)
    for t in range(S // L):
        for g in range(G):
            o = O.prefill_tile(Q[g, t * L:(t + 1) * L], K, V, list(range(t + 1)), L, t * L, 0.3)
            assert np.allclose(o, ref[g, t * L:(t + 1) * L], rtol=0, atol=1e-12)


def check_prefill_masked(seed=13, S=256, L=32, D=16):
    """A sparse chunk set per tile == fp64 SDPA with an explicit mask keeping
    the tile's chunks and the causal triangle."""
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((S, D))
    K = rng.standard_normal((S, D))
    V = rng.standard_normal((S, D))
    for t in range(S // L):
        chunks = sorted({0, t} | set(rng.choice(t + 1, size=min(t + 1, 2), replace=False).tolist()))
        mask = np.zeros((L, S), dtype=bool)
        for c in chunks:
            mask[:, c * L:(c + 1) * L] = True
        pos = t * L + np.arange(L)
        mask &= np.arange(S)[None, :] <= pos[:, None]
        ref = _sdpa(Q[None, t * L:(t + 1) * L], K[None], V[None], mask=mask[None], scale=0.5)[0]
        o = O.prefill_tile(Q[t * L:(t + 1) * L], K, V, chunks, L, t * L, 0.5)
        assert np.allclose(o, ref, rtol=0, atol=1e-12)


ALL_CHECKS = [
    check_attention_vs_sdpa, check_dense_special_case, check_empty_attention,
    check_summary_closed_form, check_score_hand_case, check_projection_closed_form,
    check_tile_mean, check_topk_golden, check_topk_vs_torch_sort, check_topk_invariants,
    check_topk_union_golden, check_topk_union_brute_force, check_per_head_scores,
    check_topp_golden, check_topp_invariants, check_hier_golden, check_hier_all_metas_is_flat,
    check_meta_linearity, check_merge_closed_form, check_partition,
    check_prefill_dense_causal, check_prefill_masked, check_hybrid_golden, check_hybrid_vs_sdpa,
    check_pipeline_topp_scale_under_projection, check_pipeline_rope_branch,
    check_rope_closed_forms, check_token_sparse_golden, check_token_sparse_invariants,
    check_token_sparse_vs_sdpa,
]
