"""Plant plausible mistakes in the CPU oracle and check that the pins catch
each one.  Every mutant is a small edit of one oracle function (a dropped
term, a wrong sign or index, a flipped comparison, a transposed operand); the
test patches it in with monkeypatch, runs the pins and expects at least one
to fail.  Nothing here touches a GPU."""
import math

import numpy as np
import pytest

import pins
from oracle import csa_oracle as O
from oracle import pipeline as OP

_orig = {name: getattr(O, name) for name in
         ["attend", "select_topk", "select_topp", "score_chunks", "lse_merge",
          "causal_attend", "meta_summaries", "chunk_summaries", "select_hier",
          "forced_set", "topp_probs", "decode_partition", "tile_mean_q",
          "select_topk_union", "score_chunks_per_head", "hybrid_unit", "rope",
          "token_importance", "coverage_budget", "select_tokens", "token_sparse_head"]}


def attend_no_scale(q, K, V, tokens, scale):
    return _orig["attend"](q, K, V, tokens, 1.0)


def attend_no_max_shift_wrong_lse(q, K, V, tokens, scale):
    o, lse = _orig["attend"](q, K, V, tokens, scale)
    return o, lse - math.log(max(len(tokens), 1)) * 0 + 1e-3  # lse off by a constant


def attend_last_token_dropped(q, K, V, tokens, scale):
    return _orig["attend"](q, K, V, tokens[:-1], scale)


def topk_ties_to_higher_index(scores, k_free, n_sink, n_local, n_valid=None):
    scores = np.asarray(scores, dtype=np.float64)
    v = len(scores) if n_valid is None else int(n_valid)
    Fs = O.forced_set(v, n_sink, n_local)
    cand = [c for c in range(v) if c not in Fs]
    order = sorted(cand, key=lambda c: (-scores[c], -c))
    return sorted(Fs | set(order[:k_free])), math.inf


def topk_forced_inside_k(scores, k_free, n_sink, n_local, n_valid=None):
    v = len(scores) if n_valid is None else int(n_valid)
    nf = len(O.forced_set(v, n_sink, n_local))
    return _orig["select_topk"](scores, max(k_free - nf, 0), n_sink, n_local, n_valid)


def topk_ascending(scores, k_free, n_sink, n_local, n_valid=None):
    return _orig["select_topk"](-np.asarray(scores, dtype=np.float64), k_free, n_sink,
                                n_local, n_valid)


def forced_local_off_by_one(n_valid, n_sink, n_local):
    s = set(range(min(n_sink, n_valid)))
    s.update(range(max(n_valid - n_local - 1, 0), n_valid - 1))
    return s


def topp_strict(scores, logit_scale, p, budget, n_sink, n_local):
    # '>' instead of '>=': nudge p up by one ulp
    return _orig["select_topp"](scores, logit_scale, np.nextafter(p, 2.0), budget, n_sink, n_local)


def topp_cap_after_union(scores, logit_scale, p, budget, n_sink, n_local):
    nf = len(O.forced_set(len(scores), n_sink, n_local))
    return _orig["select_topp"](scores, logit_scale, p, max(budget - nf, 0), n_sink, n_local)


def topp_probs_no_scale(scores, logit_scale):
    return _orig["topp_probs"](scores, 1.0)


def score_first_head_only(q, summ, Hkv, proj=None):
    q = np.array(q, dtype=np.float64)
    G = q.shape[2] // Hkv
    for h in range(Hkv):
        q[:, :, h * G + 1:(h + 1) * G] = 0.0
    return _orig["score_chunks"](q, summ, Hkv, proj)


def score_proj_transposed(q, summ, Hkv, proj=None):
    if proj is None:
        return _orig["score_chunks"](q, summ, Hkv, None)
    P = np.asarray(proj)
    PP = P @ P.T  # use the D x D Gram matrix's wrong side: q P P^T P^T ...
    qq = np.einsum("bnhd,de->bnhe", np.asarray(q, dtype=np.float64), PP / np.abs(PP).max())
    return _orig["score_chunks"](qq, summ, Hkv, proj)


def merge_plain_average(o_part, lse_part):
    o_part = np.asarray(o_part)
    lse_part = np.asarray(lse_part)
    o, lse = _orig["lse_merge"](o_part, lse_part)
    valid = lse_part > -math.inf
    avg = (o_part * valid[..., None]).sum(axis=1) / np.maximum(valid.sum(axis=1), 1)[:, None]
    return avg, lse


def merge_reads_empty(o_part, lse_part):
    lse_part = np.where(np.asarray(lse_part) == -math.inf, 0.0, lse_part)  # zero-initialised slot
    return _orig["lse_merge"](o_part, lse_part)


def causal_off_by_one(Q_rows, k, v, key_pos, q_start, scale):
    return _orig["causal_attend"](Q_rows, k, v, np.asarray(key_pos) + 1, q_start, scale)


def causal_no_mask(Q_rows, k, v, key_pos, q_start, scale):
    return _orig["causal_attend"](Q_rows, k, v, np.zeros_like(np.asarray(key_pos)), q_start, scale)


def meta_sum_not_mean(summ, Gm):
    return _orig["meta_summaries"](summ, Gm) * Gm


def summaries_first_row(K, L, proj=None):
    K = np.asarray(K, dtype=np.float64)
    T, D = K.shape[-2:]
    C = T // L
    m = K[..., : C * L, :].reshape(K.shape[:-2] + (C, L, D))[..., 0, :]
    return m if proj is None else m @ proj


def hier_forced_in_pool(q_group, meta, summ, Gm, top_meta, k_free, n_sink, n_local):
    res, a, b = _orig["select_hier"](q_group, meta, summ, Gm, top_meta, k_free, n_sink, n_local)
    Fs = O.forced_set(summ.shape[0], n_sink, n_local)
    free = [c for c in res if c not in Fs]
    return sorted(Fs | set(free[: max(k_free - len(Fs), 0)])), a, b


def hier_meta_ties_high(q_group, meta, summ, Gm, top_meta, k_free, n_sink, n_local):
    return _orig["select_hier"](q_group, meta[::-1].copy(), summ, Gm, top_meta, k_free,
                                n_sink, n_local)


def partition_ceil(n_chunks, n_parts):
    N = sum(n_chunks)
    step = -(-N // n_parts) if n_parts else N
    out, base = [], 0
    for n in n_chunks:
        spl, pos = [], 0
        while pos < n:
            nxt = min(n, pos + max(step, 1))
            spl.append((pos, nxt))
            pos = nxt
        out.append(spl)
        base += n
    return out


def tile_mean_first_row(Q, tile_m):
    Q = np.asarray(Q, dtype=np.float64)
    return Q[:, ::tile_m]


def union_is_intersection(scores_heads, k_free, n_sink, n_local, n_valid=None):
    sets = [set(_orig["select_topk"](row, k_free, n_sink, n_local, n_valid)[0])
            for row in np.asarray(scores_heads, dtype=np.float64)]
    return sorted(set.intersection(*sets)), math.inf


def union_first_head_only(scores_heads, k_free, n_sink, n_local, n_valid=None):
    return _orig["select_topk_union"](np.asarray(scores_heads)[:1], k_free, n_sink, n_local, n_valid)


def union_of_group_sum(scores_heads, k_free, n_sink, n_local, n_valid=None):
    s = np.asarray(scores_heads, dtype=np.float64).sum(axis=0, keepdims=True)
    return _orig["select_topk_union"](s, k_free, n_sink, n_local, n_valid)


def per_head_scores_group_summed(q_group, summ_unit, proj=None):
    per = _orig["score_chunks_per_head"](q_group, summ_unit, proj)
    return np.repeat(per.sum(axis=0, keepdims=True), per.shape[0], axis=0)


def hybrid_scope_swapped(q, K, V, Kg, Vg, chunks, L, scale, scope):
    other = "all" if scope == "selected" else "selected"
    return _orig["hybrid_unit"](q, K, V, Kg, Vg, chunks, L, scale, other)


def hybrid_no_gists(q, K, V, Kg, Vg, chunks, L, scale, scope):
    return O.decode_unit(q, K, V, chunks, L, scale)


def hybrid_gist_logits_unscaled(q, K, V, Kg, Vg, chunks, L, scale, scope):
    return _orig["hybrid_unit"](q, K, V, np.asarray(Kg, dtype=np.float64) / scale, Vg, chunks,
                                L, scale, scope)


def hybrid_selected_gists_shifted(q, K, V, Kg, Vg, chunks, L, scale, scope):
    # the selected scope takes the gist row of the chunk after each chosen one
    if scope != "selected":
        return _orig["hybrid_unit"](q, K, V, Kg, Vg, chunks, L, scale, scope)
    C = np.asarray(Kg).shape[0]
    nxt = [(c + 1) % C for c in range(C)]
    return _orig["hybrid_unit"](q, K, V, np.asarray(Kg, dtype=np.float64)[nxt],
                                np.asarray(Vg, dtype=np.float64)[nxt], chunks, L, scale, scope)


# decode-step composition (oracle/pipeline.py)

def topp_scale_of_rank(D):
    return 1.0 / math.sqrt(2.0)  # 1/sqrt(R) of the pin's rank-2 projection


def topp_scale_unit(D):
    return 1.0


def rope_query_at_T(T):
    return T


def stored_unrounded(x, like):
    return np.asarray(x, dtype=np.float64)


def rope_sin_sign_flipped(x, pos, theta):
    return _orig["rope"](x, -np.asarray(pos, dtype=np.float64), theta)


def rope_adjacent_pairs(x, pos, theta):
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])  # pairs (2i, 2i+1)
    inv = np.argsort(perm)
    return _orig["rope"](x[..., perm], pos, theta)[..., inv]


def rope_freq_exponent_off(x, pos, theta):
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    freq = theta ** (-1.0 * np.arange(h) / D)  # i/D instead of 2i/D
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def importance_not_causal(Q_obs, K, obs_pos, scale):
    return _orig["token_importance"](Q_obs, K, np.full(len(obs_pos), len(K)), scale)


def budget_strict(mass, tau):
    m = np.asarray(mass, dtype=np.float64)
    m = m / m.sum()
    dropped, acc = 0, 0.0
    for j in sorted(range(len(m)), key=lambda j: (m[j], -j)):
        if acc + m[j] >= tau:  # stops at equality
            break
        acc += m[j]
        dropped += 1
    return len(m) - dropped


def budget_keeps_tail(mass, tau):
    m = np.asarray(mass, dtype=np.float64)
    m = m / m.sum()
    kept, acc = 0, 0.0  # counts from the top until the kept mass reaches tau
    for j in sorted(range(len(m)), key=lambda j: (-m[j], j)):
        if acc >= tau:
            break
        acc += m[j]
        kept += 1
    return kept


def tokens_least_important(importance, k):
    return _orig["select_tokens"](-np.asarray(importance, dtype=np.float64), k)


def token_sparse_dense_rows(Q_group, K_head, V_head, tokens, scale):
    out = _orig["token_sparse_head"](Q_group, K_head, V_head, tokens, scale)
    full = _orig["token_sparse_head"](Q_group, K_head, V_head, range(len(K_head)), scale)
    keep = np.zeros(len(K_head), dtype=bool)
    keep[list(tokens)] = True
    out[~keep] = full[~keep]  # rows left out attend densely instead of 0
    return out


def token_sparse_not_causal(Q_group, K_head, V_head, tokens, scale):
    Q_group = np.asarray(Q_group, dtype=np.float64)
    S, G, D = Q_group.shape
    out = np.zeros((S, G, np.asarray(V_head).shape[-1]))
    t = np.asarray(sorted(tokens), dtype=np.int64)
    for g in range(G):
        out[t, g] = O.causal_attend(Q_group[t, g], np.asarray(K_head)[t], np.asarray(V_head)[t],
                                    np.zeros(len(t)), 0, scale)
    return out


MUTANTS = [
    ("attend", attend_no_scale),
    ("attend", attend_no_max_shift_wrong_lse),
    ("attend", attend_last_token_dropped),
    ("select_topk", topk_ties_to_higher_index),
    ("select_topk", topk_forced_inside_k),
    ("select_topk", topk_ascending),
    ("forced_set", forced_local_off_by_one),
    ("select_topp", topp_strict),
    ("select_topp", topp_cap_after_union),
    ("topp_probs", topp_probs_no_scale),
    ("score_chunks", score_first_head_only),
    ("score_chunks", score_proj_transposed),
    ("lse_merge", merge_plain_average),
    ("lse_merge", merge_reads_empty),
    ("causal_attend", causal_off_by_one),
    ("causal_attend", causal_no_mask),
    ("meta_summaries", meta_sum_not_mean),
    ("chunk_summaries", summaries_first_row),
    ("select_hier", hier_forced_in_pool),
    ("select_hier", hier_meta_ties_high),
    ("decode_partition", partition_ceil),
    ("tile_mean_q", tile_mean_first_row),
    ("select_topk_union", union_is_intersection),
    ("select_topk_union", union_first_head_only),
    ("select_topk_union", union_of_group_sum),
    ("score_chunks_per_head", per_head_scores_group_summed),
    ("hybrid_unit", hybrid_scope_swapped),
    ("hybrid_unit", hybrid_no_gists),
    ("hybrid_unit", hybrid_gist_logits_unscaled),
    ("hybrid_unit", hybrid_selected_gists_shifted),
    ("pipeline.topp_logit_scale", topp_scale_of_rank),
    ("pipeline.topp_logit_scale", topp_scale_unit),
    ("pipeline.rope_query_position", rope_query_at_T),
    ("pipeline._stored", stored_unrounded),
    ("rope", rope_sin_sign_flipped),
    ("rope", rope_adjacent_pairs),
    ("rope", rope_freq_exponent_off),
    ("token_importance", importance_not_causal),
    ("coverage_budget", budget_strict),
    ("coverage_budget", budget_keeps_tail),
    ("select_tokens", tokens_least_important),
    ("token_sparse_head", token_sparse_dense_rows),
    ("token_sparse_head", token_sparse_not_causal),
]


def _pins_fail():
    for check in pins.ALL_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


@pytest.mark.parametrize("name,mutant", MUTANTS, ids=lambda x: getattr(x, "__name__", x))
def test_mutant_is_caught(monkeypatch, name, mutant):
    if name.startswith("pipeline."):
        monkeypatch.setattr(OP, name.split(".", 1)[1], mutant)
    else:
        monkeypatch.setattr(O, name, mutant)
    # a planted mistake may leave a row with nothing visible (inf - inf):
    # that is for the pins to catch, not a warning
    with np.errstate(invalid="ignore"):
        caught = _pins_fail()
    assert caught, f"no pin caught the planted mistake {mutant.__name__}"


def test_unmutated_oracle_passes():
    assert not _pins_fail()
