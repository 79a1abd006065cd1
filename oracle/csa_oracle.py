"""CPU oracle for query-adaptive chunk-sparse attention (fp64, plain numpy).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this module.  The CUDA
library never calls it and shares no code with it.

What it computes, in the order the pages give it:

* Chunking and summary keys.  The SSA summary (aitrends.kr/articles/69798,
  section "기술 상세" / technical details) splits the sequence into chunks of
  length L, each with one summary key; the HiLS review ("Hierarchical Sparse
  Attention Done Right", section 1, "Landmark Token") summarises a chunk by one
  key as well.  The learned gist / landmark keys need trained weights, so the
  stand-in summary is the mean of the chunk's keys.  The RTPurbo review ("Full
  Attention Strikes Back", section 1, "Low-dimensional Projection") scores on a
  16-dim projection of the keys; the projected summary is P^T times the mean.
* Relevance score.  SSA summary, section "방법론" (method): s_{t,m} = q_t^T k_{g_m},
  the inner product of the current query with each chunk's summary key.  For
  GQA the HiLS review (section 1, "GQA") selects chunks per query-head group;
  the score of a KV head is the sum over its query heads.
* Selection.  Top-k over chunk scores (SSA summary, "핵심 기여" / contributions
  and "방법론"); dynamic top-p that keeps the smallest prefix securing a target
  attention mass (RTPurbo review, section 1, "Dynamic Top-p Selection"); the
  coarse-to-fine gist-of-gist selection (SSA summary, "핵심 기여", H-SSA and the
  glossary entry "Hierarchical Gist-of-Gist").  Sink and local chunks are
  always kept.
* Exact attention over the raw KV of the selected chunks (SSA summary,
  "방법론": standard attention over the hybrid context), and over the hybrid
  context itself: the gist KV and the raw KV of the selected chunks
  ("방법론", "기술 상세"), or, read from the glossary entry "Selective
  Unfolding", the gist KV of every chunk plus the raw KV of the selected
  ones; computed as split-K
  partials combined afterwards (SSA summary, "핵심 기여": compact index list and
  split-K partial attention).
* Block-sparse causal prefill over per-query-tile chunk sets (SSA summary,
  "핵심 기여": block-skip prefill; HiLS review, section 3: adjacent queries
  grouped into one union of chunks).

Readings taken where the pages are silent (each one is listed with its
reason in the design notes): summaries are chunk means; forced chunks are
kept outside the top-k pool; the top-p softmax is over all chunks of the
unit with logit scale 1/sqrt(D), the prefix is minimal with cum >= p, the cap
applies to the prefix and the forced chunks are added afterwards; ties in any
ordering go to the lower chunk index; a hierarchical meta-summary is the mean
of its children's summaries and forced chunks play no part at meta level.

Every function takes numpy arrays (converted by the caller from the input
tensors; bf16 values are exact in fp64) and works in float64.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -math.inf


# ---------------------------------------------------------------- summaries

def chunk_summaries(K: np.ndarray, L: int, proj: np.ndarray | None = None) -> np.ndarray:
    """Summary key per chunk: mean of the chunk's L key rows, optionally
    projected to P^T * mean (RTPurbo review, section 1, low-dimensional
    projection).

    K: [..., T, D] -> [..., T // L, D] (or [..., T // L, R] with proj [D, R]).
    """
    K = np.asarray(K, dtype=np.float64)
    T, D = K.shape[-2:]
    C = T // L
    mean = K[..., : C * L, :].reshape(K.shape[:-2] + (C, L, D)).mean(axis=-2)
    if proj is not None:
        mean = mean @ np.asarray(proj, dtype=np.float64)
    return mean


def meta_summaries(summ: np.ndarray, Gm: int) -> np.ndarray:
    """Meta-summary of each group of Gm consecutive chunks: the mean of their
    summaries (stand-in for the meta-gist token of H-SSA, SSA summary,
    glossary "Hierarchical Gist-of-Gist").  [..., C, Ds] -> [..., C // Gm, Ds]."""
    summ = np.asarray(summ, dtype=np.float64)
    C, Ds = summ.shape[-2:]
    M = C // Gm
    return summ[..., : M * Gm, :].reshape(summ.shape[:-2] + (M, Gm, Ds)).mean(axis=-2)


def tile_mean_q(Q: np.ndarray, tile_m: int) -> np.ndarray:
    """Mean query of each tile of tile_m consecutive positions, per head: the
    representative of the adjacent queries that share one chunk union (HiLS
    review, section 3, union chunks).  Q [B, S, Hq, D] -> [B, S // tile_m, Hq, D]."""
    Q = np.asarray(Q, dtype=np.float64)
    B, S, Hq, D = Q.shape
    n = S // tile_m
    return Q[:, : n * tile_m].reshape(B, n, tile_m, Hq, D).mean(axis=2)


# ------------------------------------------------------------------- scores

def score_chunks(q: np.ndarray, summ: np.ndarray, Hkv: int,
                 proj: np.ndarray | None = None) -> np.ndarray:
    """Relevance of every chunk for every query row and KV head.

    S[b, h, n, c] = sum over the query heads g of KV head h of  q~[b, n, g] . summ[b, h, c],
    with q~ = P^T q when a projection is given (SSA summary, "방법론":
    s = q^T k_gist; HiLS review, section 1: group-level selection for GQA).

    q: [B, Nq, Hq, D]; summ: [B, Hkv, C, Ds] -> [B, Hkv, Nq, C].
    """
    q = np.asarray(q, dtype=np.float64)
    summ = np.asarray(summ, dtype=np.float64)
    B, Nq, Hq, D = q.shape
    G = Hq // Hkv
    C = summ.shape[2]
    out = np.zeros((B, Hkv, Nq, C), dtype=np.float64)
    for b in range(B):
        for h in range(Hkv):
            for g in range(G):
                qg = q[b, :, h * G + g, :]  # [Nq, D]
                if proj is not None:
                    qg = qg @ np.asarray(proj, dtype=np.float64)  # [Nq, R]
                out[b, h] += qg @ summ[b, h].T  # per-head inner products, summed
    return out


# ---------------------------------------------------------------- selection

def forced_set(n_valid: int, n_sink: int, n_local: int) -> set:
    """Chunks a unit always keeps: the first n_sink (attention sink) and the
    last n_local of the chunks it can see ([0, n_valid))."""
    s = set(range(min(n_sink, n_valid)))
    s.update(range(max(n_valid - n_local, 0), n_valid))
    return s


def _rank_order(values, candidates):
    """Candidates ordered by value descending, lower chunk index first on ties."""
    return sorted(candidates, key=lambda c: (-float(values[c]), c))


def select_topk(scores: np.ndarray, k_free: int, n_sink: int, n_local: int,
                n_valid: int | None = None) -> tuple[list, float]:
    """Top-k chunk set of one unit (SSA summary, "방법론": the k highest-scoring
    chunks are unfolded).

    The unit sees chunks [0, n_valid).  Result = forced set  U  the k_free best
    of the remaining chunks by (score desc, index asc), returned ascending.
    Also returns the relative score gap at the cut, for near-tie reporting:
    |s_(k) - s_(k+1)| / max(|s_(k)|, |s_(k+1)|) (inf when there is no cut)."""
    scores = np.asarray(scores, dtype=np.float64)
    v = len(scores) if n_valid is None else int(n_valid)
    F = forced_set(v, n_sink, n_local)
    cand = [c for c in range(v) if c not in F]
    order = _rank_order(scores, cand)
    chosen = order[:k_free]
    gap = math.inf
    if 0 < k_free < len(order):
        a, b = scores[order[k_free - 1]], scores[order[k_free]]
        gap = abs(a - b) / max(abs(a), abs(b), 1e-30)
    return sorted(F | set(chosen)), gap


def score_chunks_per_head(q_group: np.ndarray, summ_unit: np.ndarray,
                          proj: np.ndarray | None = None) -> np.ndarray:
    """Relevance of every chunk for each query head of one unit, without the
    group sum: S[g, c] = q~_g . summ[c] (SSA summary, "방법론": s = q^T k_gist,
    evaluated per query head).  q_group [G, D]; summ_unit [C, Ds] -> [G, C]."""
    q = np.asarray(q_group, dtype=np.float64)
    if proj is not None:
        q = q @ np.asarray(proj, dtype=np.float64)
    return q @ np.asarray(summ_unit, dtype=np.float64).T


def select_topk_union(scores_heads: np.ndarray, k_free: int, n_sink: int, n_local: int,
                      n_valid: int | None = None) -> tuple[list, float]:
    """Per-head top-k with the GQA union (SSA summary, glossary entry
    "Grouped-Query Attention": every query head makes its own top-k choice and
    the group loads the union of the chosen chunks once).

    scores_heads [G, C]: each head's own top-k (forced set plus its k_free best
    non-forced chunks, select_topk); the result is the ascending union over
    the heads.  The returned gap is the smallest of the heads' boundary gaps."""
    out, gap = set(), math.inf
    for row in np.asarray(scores_heads, dtype=np.float64):
        chunks, g = select_topk(row, k_free, n_sink, n_local, n_valid)
        out.update(chunks)
        gap = min(gap, g)
    return sorted(out), gap


def topp_probs(scores: np.ndarray, logit_scale: float) -> np.ndarray:
    """Chunk-level attention mass pi_c = softmax(S_c * logit_scale) over all
    chunks of the unit: the first-order chunk-mass estimate of the HiLS review
    (section 1, "Chunk Mass Surrogate") with the chunk summary standing in for
    the chunk's keys."""
    z = np.asarray(scores, dtype=np.float64) * logit_scale
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def select_topp(scores: np.ndarray, logit_scale: float, p: float, budget: int,
                n_sink: int, n_local: int) -> tuple[list, int, float]:
    """Dynamic top-p chunk set of one unit (RTPurbo review, section 1: a
    query-dependent number of chunks that secures the attention mass).

    Chunks sorted by (pi desc, index asc); n_p = the smallest n whose prefix
    mass reaches p (cum >= p); the prefix is cut at min(n_p, budget) and the
    forced chunks are added.  Returns (ascending set, n_p, gap), where gap is
    the smaller of the relative pi gap at the cut and |cum_{n_p-1} - p| / p."""
    pi = topp_probs(scores, logit_scale)
    C = len(pi)
    order = _rank_order(pi, range(C))
    cum = 0.0
    n_p = C
    cum_before = 0.0
    for n, c in enumerate(order, start=1):
        cum_before = cum
        cum += pi[c]
        if cum >= p:
            n_p = n
            break
    n_take = min(n_p, budget)
    T = order[:n_take]
    gap = math.inf
    if 0 < n_take < C:
        a, b = pi[order[n_take - 1]], pi[order[n_take]]
        gap = abs(a - b) / max(abs(a), abs(b), 1e-300)
    if n_p <= budget:
        gap = min(gap, abs(cum_before - p) / p, abs(cum - p) / p)
    F = forced_set(C, n_sink, n_local)
    return sorted(F | set(T)), n_p, gap


def select_hier(q_group: np.ndarray, meta: np.ndarray, summ: np.ndarray, Gm: int,
                top_meta: int, k_free: int, n_sink: int, n_local: int
                ) -> tuple[list, float, float]:
    """Two-level coarse-to-fine selection of one unit (SSA summary, "핵심 기여":
    H-SSA narrows candidate segments with meta-gists, then re-scores the gists
    inside them).

    q_group [G, D] are the unit's query heads; meta [M, D], summ [C, D].
    Meta scores and child scores are the group-summed inner products.  Keep
    the top_meta metas by (score desc, index asc); among their children that
    are not forced, keep the k_free best; add the forced chunks.
    Returns (ascending set, meta-cut gap, child-cut gap)."""
    qg = np.asarray(q_group, dtype=np.float64)
    meta = np.asarray(meta, dtype=np.float64)
    summ = np.asarray(summ, dtype=np.float64)
    M = meta.shape[0]
    C = summ.shape[0]
    ms = np.zeros(M)
    for g in range(qg.shape[0]):
        ms += meta @ qg[g]
    morder = _rank_order(ms, range(M))
    metas = morder[:top_meta]
    mgap = math.inf
    if 0 < top_meta < M:
        a, b = ms[morder[top_meta - 1]], ms[morder[top_meta]]
        mgap = abs(a - b) / max(abs(a), abs(b), 1e-30)
    F = forced_set(C, n_sink, n_local)
    children = [c for m in metas for c in range(m * Gm, (m + 1) * Gm) if c not in F]
    cs = np.zeros(C)
    for g in range(qg.shape[0]):
        cs[children] += summ[children] @ qg[g]
    corder = _rank_order(cs, children)
    chosen = corder[:k_free]
    cgap = math.inf
    if 0 < k_free < len(corder):
        a, b = cs[corder[k_free - 1]], cs[corder[k_free]]
        cgap = abs(a - b) / max(abs(a), abs(b), 1e-30)
    return sorted(F | set(chosen)), mgap, cgap


# ---------------------------------------------------------------- attention

def chunk_tokens(chunks, L: int) -> np.ndarray:
    """Token positions of the given chunks, in chunk order."""
    if len(chunks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(c * L, (c + 1) * L) for c in chunks])


def attend(q_heads: np.ndarray, K: np.ndarray, V: np.ndarray, tokens: np.ndarray,
           scale: float) -> tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of each query head over the given key tokens
    (SSA summary, "방법론": standard attention over the unfolded raw KV).

    a_j = scale * q . k_j;  o = sum_j softmax(a)_j v_j;  lse = log sum_j exp(a_j).
    Two passes in fp64: the max, then the normalised sum.  An empty token set
    gives o = 0 and lse = -inf.
    q_heads [G, D], K/V [T, D] -> o [G, D], lse [G]."""
    qh = np.asarray(q_heads, dtype=np.float64)
    G, D = qh.shape
    if len(tokens) == 0:
        return np.zeros((G, V.shape[-1])), np.full(G, NEG_INF)
    k = np.asarray(K[tokens], dtype=np.float64)
    v = np.asarray(V[tokens], dtype=np.float64)
    a = (qh @ k.T) * scale  # [G, n]
    m = a.max(axis=1, keepdims=True)
    w = np.exp(a - m)
    l = w.sum(axis=1, keepdims=True)
    o = (w @ v) / l
    lse = m[:, 0] + np.log(l[:, 0])
    return o, lse


def decode_unit(q_group, K_unit, V_unit, chunks, L: int, scale: float):
    """Attention of one unit's query heads over the raw KV of its chunk set."""
    return attend(q_group, K_unit, V_unit, chunk_tokens(sorted(chunks), L), scale)


def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotary position embedding of rows x [..., n, D] at positions pos
    (broadcast against the row axis), rotate-half pairing: for i < D/2 the
    pair (x_i, x_{i+D/2}) turns by the angle pos * theta^(-2i/D).

    The RTPurbo review (section 1, "Low-dimensional Projection") scores on a
    projection taken before RoPE because RoPE makes scores depend on the
    distance; the pages do not write RoPE out, so this is the common
    rotate-half form with base theta."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    freq = theta ** (-2.0 * np.arange(h) / D)                      # [h]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq      # [..., n, h]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


GIST_SCOPES = ("selected", "all")


def hybrid_unit(q_group, K_unit, V_unit, Kg_unit, Vg_unit, chunks, L: int, scale: float,
                scope: str):
    """Attention of one unit's query heads over its hybrid context (SSA
    summary, "방법론" and "기술 상세").

    scope = "selected" (the method and technical-details sections): the top-k
    chunks I_t are the only ones brought back, each with its gist KV and its
    raw KV; K_hybrid / V_hybrid are the union of the gist rows and the raw
    rows of the chunks in I_t.
    scope = "all" (the glossary entry "Selective Unfolding" read as the
    context): the gist row of every chunk stays in the context and the raw
    rows of the chunks in I_t are added next to them.

    One softmax runs over the union, with the same scale for gist and raw
    logits.  K_unit/V_unit [T, D] raw; Kg_unit/Vg_unit [C, D], one gist
    key/value per chunk -> o [G, D], lse [G]."""
    if scope not in GIST_SCOPES:
        raise ValueError(f"gist scope {scope!r}")
    sel = sorted(chunks)
    tok = chunk_tokens(sel, L)
    Kg = np.asarray(Kg_unit, dtype=np.float64)
    Vg = np.asarray(Vg_unit, dtype=np.float64)
    gist_rows = np.asarray(sel, dtype=np.int64) if scope == "selected" else np.arange(Kg.shape[0])
    Kr = np.asarray(K_unit, dtype=np.float64)[tok]
    Vr = np.asarray(V_unit, dtype=np.float64)[tok]
    Kh = np.concatenate([Kr, Kg[gist_rows]], axis=0)
    Vh = np.concatenate([Vr, Vg[gist_rows]], axis=0)
    return attend(q_group, Kh, Vh, np.arange(Kh.shape[0]), scale)


def lse_merge(o_part: np.ndarray, lse_part: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Combine split-K partials of one or more rows (SSA summary, "핵심 기여":
    split-K partial attention combined afterwards).

    lse = log sum_s exp(lse_s);  o = sum_s exp(lse_s - lse) o_s.  A split with
    lse = -inf holds no tokens and contributes nothing (its o is not read).
    o_part [R, S, D], lse_part [R, S] -> o [R, D], lse [R]."""
    o_part = np.asarray(o_part, dtype=np.float64)
    lse_part = np.asarray(lse_part, dtype=np.float64)
    R, S, D = o_part.shape
    out = np.zeros((R, D))
    lse = np.full(R, NEG_INF)
    for r in range(R):
        valid = [s for s in range(S) if lse_part[r, s] != NEG_INF]
        if not valid:
            continue
        mx = max(lse_part[r, s] for s in valid)
        tot = sum(math.exp(lse_part[r, s] - mx) for s in valid)
        lse[r] = mx + math.log(tot)
        for s in valid:
            out[r] += math.exp(lse_part[r, s] - lse[r]) * o_part[r, s]
    return out, lse


def decode_partition(n_chunks: list, n_parts: int) -> list:
    """Split-K layout of the library's decode call, restated from its contract.

    The units' chunk lists are laid end to end (unit-major), N chunks in all,
    and cut into n_parts pieces; piece c is [floor(c*N/P), floor((c+1)*N/P)).
    Split s of unit u is its s-th non-empty intersection with a piece, in piece
    order.  Returns, per unit, a list of (begin, end) positions into the unit's
    own chunk list."""
    N = sum(n_chunks)
    P = n_parts
    bounds = [(c * N) // P for c in range(P + 1)]
    out = []
    base = 0
    for n in n_chunks:
        spl = []
        for c in range(P):
            lo, hi = max(bounds[c], base), min(bounds[c + 1], base + n)
            if lo < hi:
                spl.append((lo - base, hi - base))
        out.append(spl)
        base += n
    return out


def causal_attend(Q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, key_pos: np.ndarray,
                  q_start: int, scale: float) -> np.ndarray:
    """Causal softmax attention of query rows at positions q_start + i over
    keys at positions key_pos: row i sees key j iff key_pos[j] <= q_start + i.
    Q_rows [m, D], k/v [n, D] -> O [m, D] (zeros when n == 0)."""
    qt = np.asarray(Q_rows, dtype=np.float64)
    m = qt.shape[0]
    if len(key_pos) == 0:
        return np.zeros((m, v.shape[-1]))
    a = (qt @ np.asarray(k, dtype=np.float64).T) * scale  # [m, n]
    qpos = q_start + np.arange(m)
    a = np.where(np.asarray(key_pos)[None, :] <= qpos[:, None], a, NEG_INF)
    mx = a.max(axis=1, keepdims=True)
    w = np.exp(a - mx)
    return (w @ np.asarray(v, dtype=np.float64)) / w.sum(axis=1, keepdims=True)


def prefill_tile(Q_tile: np.ndarray, K_head: np.ndarray, V_head: np.ndarray, chunks,
                 L: int, q_start: int, scale: float) -> np.ndarray:
    """Causal attention of one query tile of one head over the raw KV of the
    tile's chunk set (SSA summary, "핵심 기여": block-sparse prefill that skips
    unselected blocks; the diagonal chunk is causally masked).

    Row i (absolute position q_start + i) sees the key tokens of the chunks
    whose position is <= q_start + i.  Q_tile [m, D] -> O [m, D]."""
    tok = chunk_tokens(sorted(chunks), L)
    return causal_attend(Q_tile, np.asarray(K_head)[tok], np.asarray(V_head)[tok], tok,
                         q_start, scale)


# ------------------------------------------------------ token-level sparsity

def token_importance(Q_obs: np.ndarray, K: np.ndarray, obs_pos: np.ndarray,
                     scale: float) -> np.ndarray:
    """Importance of every key of one KV head from a proxy attention map of
    the recent queries (Token Sparse Attention summary, section 2, "동적 토큰
    커버리지": recent queries against all keys, scores summed over the query
    axis of the attention weights).

    Q_obs [r, D]: the recent query rows of the KV head's query heads (the GQA
    group, reading: one importance per KV head, summed over its query heads);
    obs_pos [r]: their positions.  Row i attends causally (key j <= obs_pos[i])
    with softmax(scale * q.k); the importance of key j is the sum over the rows
    of its weight.  K [S, D] -> [S]."""
    q = np.asarray(Q_obs, dtype=np.float64)
    k = np.asarray(K, dtype=np.float64)
    a = (q @ k.T) * scale                                   # [r, S]
    S = k.shape[0]
    vis = np.arange(S)[None, :] <= np.asarray(obs_pos)[:, None]
    a = np.where(vis, a, NEG_INF)
    w = np.exp(a - a.max(axis=1, keepdims=True))
    w /= w.sum(axis=1, keepdims=True)
    return w.sum(axis=0)


def coverage_budget(mass: np.ndarray, tau: float) -> int:
    """Dynamic Token Coverage budget (Token Sparse Attention summary, section
    2): sort the tokens by importance ascending and drop them from the least
    important while the dropped mass stays <= tau; the budget is the number
    of tokens left.  mass [S], normalised here to sum 1; ties in the order go
    to the higher index first (so the lower index is kept)."""
    m = np.asarray(mass, dtype=np.float64)
    m = m / m.sum()
    order = sorted(range(len(m)), key=lambda j: (m[j], -j))   # ascending mass
    dropped, acc = 0, 0.0
    for j in order:
        if acc + m[j] > tau:
            break
        acc += m[j]
        dropped += 1
    return len(m) - dropped


def select_tokens(importance: np.ndarray, k: int) -> list:
    """The k most important tokens of one KV head (score desc, lower index
    first on ties), ascending: each head keeps its own top-k under the global
    budget (Token Sparse Attention summary, section 2, "헤드별 선택")."""
    return sorted(_rank_order(np.asarray(importance, dtype=np.float64),
                              range(len(importance)))[:k])


def token_sparse_head(Q_group: np.ndarray, K_head: np.ndarray, V_head: np.ndarray, tokens,
                      scale: float) -> np.ndarray:
    """Compress, attend, decompress for one KV head (Token Sparse Attention
    summary, section 2, "핵심 아키텍처"): gather the query rows of the group's
    heads and the key/value rows at the selected tokens (ascending), run dense
    causal attention on the compressed sequence, and scatter the outputs back
    to their positions of a zero output.  Q_group [S, G, D], K/V [S, D] ->
    O [S, G, D]."""
    Q_group = np.asarray(Q_group, dtype=np.float64)
    S, G, D = Q_group.shape
    out = np.zeros((S, G, np.asarray(V_head).shape[-1]))
    t = np.asarray(sorted(tokens), dtype=np.int64)
    if len(t) == 0:
        return out
    k, v = np.asarray(K_head, dtype=np.float64)[t], np.asarray(V_head, dtype=np.float64)[t]
    for g in range(G):
        # compressed index i sees compressed j <= i: positions stay in order
        out[t, g] = causal_attend(Q_group[t, g], k, v, np.arange(len(t)), 0, scale)
    return out
