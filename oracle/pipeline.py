"""Whole-step oracle drivers: a decode step (summaries -> scores -> selection ->
attention) and a block-sparse causal prefill, per unit, in fp64.

TEST INFRASTRUCTURE (see ``oracle/csa_oracle.py``).  Inputs are torch tensors
or numpy arrays; they are converted to fp64 on the host unit by unit so that a
1M-token cache never has to exist in fp64 all at once.
"""
from __future__ import annotations

import math

import numpy as np

from . import csa_oracle as O


def to_np(x) -> np.ndarray:
    """fp64 numpy copy of a torch tensor (any device/dtype) or array."""
    if hasattr(x, "detach"):
        import torch  # conversion only
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def unit_summaries(K_unit, L: int, proj=None, block_chunks: int = 2048) -> np.ndarray:
    """Chunk summaries of one unit's keys [T, D], computed block by block."""
    T = K_unit.shape[0]
    C = T // L
    parts = []
    for c0 in range(0, C, block_chunks):
        c1 = min(C, c0 + block_chunks)
        parts.append(O.chunk_summaries(to_np(K_unit[c0 * L: c1 * L]), L, proj))
    return np.concatenate(parts, axis=0)


def topp_logit_scale(D: int) -> float:
    """Logit scale of the top-p chunk softmax: 1/sqrt(D), D the attention
    head dimension, also when the scores come from a low-rank projection.
    Reading: the HiLS review's chunk-mass surrogate (section 1) makes a
    chunk's attention mass proportional to exp(q . k_mean / sqrt(D)); the
    projected score stands in for q . k_mean (the Gaussian projection keeps
    inner products in expectation), so the attention's own scale applies."""
    return 1.0 / math.sqrt(D)


def rope_query_position(T: int) -> int:
    """Position of the decoding query in a context of T cached tokens: the
    context's last token, T - 1 (the current token's key is the last row of
    the cache)."""
    return T - 1


def decode_step(q, K, V, *, L: int, scale: float, select: str, n_sink: int, n_local: int,
                k_free: int = 0, proj=None, p: float = 0.0, budget: int = 0,
                full_heads=(), Gm: int = 0, top_meta: int = 0, units=None,
                with_attention: bool = True, gist=None, gist_scope: str = "",
                rope_theta: float = 0.0) -> dict:
    """One decode step of the units (b, kvh) listed (default: all).

    q [B, Hq, D]; K, V [B, Hkv, T, D].  Returns a dict with, per unit, the
    ascending chunk set, the boundary gap(s), n_p for top-p, and when
    ``with_attention`` the output rows o [G, D] and lse [G].  gist = (Kg, Vg),
    each [B, Hkv, T // L, D]: the sparse units attend over the hybrid context
    of ``gist_scope`` ("selected": gist and raw rows of the chosen chunks;
    "all": every chunk's gist row plus the raw rows of the chosen chunks;
    ``hybrid_unit``).
    rope_theta > 0: the RoPE-aware split (RTPurbo review, section 1): q and K
    are the pre-RoPE ones and score as they are; attention runs on the
    rotated query (at ``rope_query_position``) and keys (positions 0 .. T - 1),
    each stored in the cache's dtype as a decode step would hold them."""
    B, Hkv, T, D = K.shape
    Hq = q.shape[1]
    G = Hq // Hkv
    C = T // L
    projn = None if proj is None else to_np(proj)
    if units is None:
        units = [(b, h) for b in range(B) for h in range(Hkv)]
    res = {"sets": {}, "gap": {}, "n_p": {}, "o": {}, "lse": {}}
    for (b, h) in units:
        qg = to_np(q[b, h * G:(h + 1) * G])  # [G, D]
        if h in tuple(full_heads):
            chunks, gap = list(range(C)), math.inf
        elif select == "topk":
            summ = unit_summaries(K[b, h], L, projn)
            s = O.score_chunks(qg[None, None], summ[None, None], 1, projn)[0, 0, 0]
            chunks, gap = O.select_topk(s, k_free, n_sink, n_local)
        elif select == "topk_union":
            summ = unit_summaries(K[b, h], L, projn)
            s = O.score_chunks_per_head(qg, summ, projn)
            chunks, gap = O.select_topk_union(s, k_free, n_sink, n_local)
        elif select == "topp":
            summ = unit_summaries(K[b, h], L, projn)
            s = O.score_chunks(qg[None, None], summ[None, None], 1, projn)[0, 0, 0]
            chunks, n_p, gap = O.select_topp(s, topp_logit_scale(D), p, budget, n_sink, n_local)
            res["n_p"][(b, h)] = n_p
        elif select == "hier":
            summ = unit_summaries(K[b, h], L)
            meta = O.meta_summaries(summ, Gm)
            chunks, mgap, cgap = O.select_hier(qg, meta, summ, Gm, top_meta, k_free,
                                               n_sink, n_local)
            gap = min(mgap, cgap)
        else:
            raise ValueError(select)
        res["sets"][(b, h)] = chunks
        res["gap"][(b, h)] = gap
        if with_attention and rope_theta > 0:
            tok = O.chunk_tokens(chunks, L)
            qr = _stored(O.rope(qg, np.full(G, rope_query_position(T)), rope_theta), q)
            Kr = _stored(O.rope(to_np(K[b, h][_index(K, tok)]), tok, rope_theta), K)
            o, lse = O.attend(qr, Kr, to_np(V[b, h][_index(V, tok)]), np.arange(len(tok)), scale)
            res["o"][(b, h)] = o
            res["lse"][(b, h)] = lse
        elif with_attention and gist is not None and h not in tuple(full_heads):
            o, lse = O.hybrid_unit(qg, to_np(K[b, h]), to_np(V[b, h]), to_np(gist[0][b, h]),
                                   to_np(gist[1][b, h]), chunks, L, scale, gist_scope)
            res["o"][(b, h)] = o
            res["lse"][(b, h)] = lse
        elif with_attention:
            tok = O.chunk_tokens(chunks, L)
            Kt = to_np(K[b, h][_index(K, tok)])
            Vt = to_np(V[b, h][_index(V, tok)])
            o, lse = O.attend(qg, Kt, Vt, np.arange(len(tok)), scale)
            res["o"][(b, h)] = o
            res["lse"][(b, h)] = lse
    return res


def _stored(x: np.ndarray, like) -> np.ndarray:
    """x rounded to the element type of `like`, as fp64: a bf16 cache holds
    its rotated keys (and the rotated query) in bf16, as a post-RoPE KV cache
    does.  torch's round-to-nearest-even conversion is the library step."""
    if hasattr(like, "dtype") and str(like.dtype) == "torch.bfloat16":
        import torch
        return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _index(t, idx: np.ndarray):
    """An index array usable on t's framework (torch tensors need a tensor)."""
    if hasattr(t, "detach"):
        import torch
        return torch.as_tensor(idx, dtype=torch.long, device=t.device)
    return idx


def prefill_units(Q, K, V, *, tile_m: int, L: int, scale: float, k_free: int,
                  n_sink: int, n_local: int, units, with_attention: bool = True) -> dict:
    """Block-sparse causal prefill for the listed units (b, t, kvh).

    Per unit: tile-mean query of each head of the group, group-summed scores
    against the summaries of the causally visible chunks [0, n_valid) with
    n_valid = ((t + 1) * tile_m - 1) // L + 1, top-k with the sink and the
    diagonal chunk forced, then causal attention of the tile's rows.
    Returns sets, gaps and O [G, tile_m, D] per unit."""
    B, S, Hq, D = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    summ_cache = {}
    res = {"sets": {}, "gap": {}, "O": {}}
    for (b, t, h) in units:
        if (b, h) not in summ_cache:
            summ_cache[(b, h)] = unit_summaries(K[b, h], L)
        summ = summ_cache[(b, h)]
        Qt = to_np(Q[b, t * tile_m:(t + 1) * tile_m, h * G:(h + 1) * G])  # [m, G, D]
        qbar = O.tile_mean_q(Qt[None], tile_m)[0, 0]  # [G, D]
        n_valid = ((t + 1) * tile_m - 1) // L + 1
        s = O.score_chunks(qbar[None, None], summ[None, None, :n_valid], 1)[0, 0, 0]
        chunks, gap = O.select_topk(s, k_free, n_sink, n_local, n_valid=n_valid)
        res["sets"][(b, t, h)] = chunks
        res["gap"][(b, t, h)] = gap
        if with_attention:
            tok = O.chunk_tokens(chunks, L)
            Kt = to_np(K[b, h][_index(K, tok)])
            Vt = to_np(V[b, h][_index(V, tok)])
            outs = []
            for g in range(G):
                outs.append(O.causal_attend(Qt[:, g], Kt, Vt, tok, t * tile_m, scale))
            res["O"][(b, t, h)] = np.stack(outs)
    return res

