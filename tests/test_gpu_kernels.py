"""Per-call parity of the CUDA library against the CPU oracle, through the C
ABI, on seeded inputs that span several tiles and a ragged tail, plus the
edge cases (empty and one-element sets, n_valid = 0/1, ties, more pieces
than chunks, group sizes 1..8, both head dims and chunk lengths)."""
import math

import numpy as np
import pytest
import torch

import parity
from oracle import csa_oracle as O
from oracle.pipeline import to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from query_adaptive_chunk_b200 import csa as mod
    return mod


def _gen(seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return g


def _randn(shape, seed, dtype=torch.float32):
    return torch.randn(shape, generator=_gen(seed), device="cuda").to(dtype)


def _dt(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


# ---------------------------------------------------------------- precompute

@pytest.mark.parametrize("dtype,D,L,R", [("f32", 64, 64, 0), ("bf16", 128, 64, 0),
                                         ("bf16", 128, 128, 16), ("bf16", 64, 128, 32),
                                         ("f32", 128, 64, 128)])
def test_chunk_summaries(csa, dtype, D, L, R):
    B, Hkv, C = 2, 3, 7
    K = _randn((B, Hkv, C * L, D), 1, _dt(dtype))
    P = _randn((D, R), 2) / 4 if R else None
    Ds = R if R else D
    out = torch.empty(B, Hkv, C, Ds, device="cuda")
    csa.csa_chunk_summaries(K, K.dtype, B, Hkv, C * L, D, L, P, R, out)
    ref = O.chunk_summaries(to_np(K), L, None if P is None else to_np(P))
    assert np.abs(out.cpu().double().numpy() - ref).max() < 1e-5


def test_tile_mean_fp32_ragged_tile(csa):
    """fp32 queries and a tile length that is not a multiple of the kernel's
    8-row batches."""
    Q = _randn((1, 12 * 7, 4, 64), 61)
    qbar = torch.empty(1, 7, 4, 64, device="cuda")
    csa.csa_tile_mean_q(Q, Q.dtype, 1, 12 * 7, 4, 64, 12, qbar)
    assert np.abs(qbar.cpu().double().numpy() - O.tile_mean_q(to_np(Q), 12)).max() < 1e-5


def test_meta_summaries_and_tile_mean(csa):
    summ = _randn((2, 3, 64, 128), 3)
    meta = torch.empty(2, 3, 8, 128, device="cuda")
    csa.csa_meta_summaries(summ, 2, 3, 64, 128, 8, meta)
    assert np.abs(meta.cpu().double().numpy() - O.meta_summaries(to_np(summ), 8)).max() < 1e-6
    Q = _randn((2, 320, 8, 64), 4, torch.bfloat16)
    qbar = torch.empty(2, 5, 8, 64, device="cuda")
    csa.csa_tile_mean_q(Q, Q.dtype, 2, 320, 8, 64, 64, qbar)
    assert np.abs(qbar.cpu().double().numpy() - O.tile_mean_q(to_np(Q), 64)).max() < 1e-5


# ---------------------------------------------------------------- scores

@pytest.mark.parametrize("G,D,R,C,causal", [(4, 128, 0, 517, False), (4, 128, 16, 1029, False),
                                            (1, 64, 0, 70, False), (8, 128, 32, 300, False),
                                            (4, 128, 0, 96, True), (2, 64, 0, 150, True)])
def test_score_chunks(csa, G, D, R, C, causal):
    B, Hkv = 2, 3
    Hq = G * Hkv
    Nq = 96 if causal else 1
    q = _randn((B, Nq, Hq, D), 5, torch.bfloat16 if not causal else torch.float32)
    P = _randn((D, R), 6) / 4 if R else None
    Ds = R if R else D
    summ = _randn((B, Hkv, C, Ds), 7) * 0.2
    full = torch.tensor([0, 1, 0], dtype=torch.uint8, device="cuda")
    scores = torch.full((B, Hkv, Nq, C), 12345.0, device="cuda")
    csa.csa_score_chunks(q, q.dtype, P, R, summ, B, Nq, Hq, Hkv, D, C, None if causal else full,
                         64 if causal else 0, 64 if causal else 0, scores)
    got = scores.cpu().double().numpy()
    ref = O.score_chunks(to_np(q), to_np(summ), Hkv, None if P is None else to_np(P))
    for b in range(B):
        for h in range(Hkv):
            if not causal and h == 1:
                assert np.all(got[b, h] == 12345.0)  # full head: row not written
                continue
            for n in range(Nq):
                vis = min(C, n + 1) if causal else C
                assert np.allclose(got[b, h, n, :vis], ref[b, h, n, :vis], rtol=1e-5, atol=1e-4)
                assert np.all(np.isneginf(got[b, h, n, vis:]))


# ---------------------------------------------------------------- top-k

def _run_topk(csa, scores, k_free, n_sink, n_local, n_valid=None, kmax=None):
    U, C = scores.shape
    kmax = kmax or max(1, min(C, k_free + n_sink + n_local))
    idx = torch.full((U, kmax), 777, dtype=torch.int32, device="cuda")
    cnt = torch.full((U,), 777, dtype=torch.int32, device="cuda")
    nv = None if n_valid is None else torch.tensor(n_valid, dtype=torch.int32, device="cuda")
    csa.csa_select_topk(scores, U, C, nv, k_free, n_sink, n_local, idx, cnt, kmax)
    return parity.gpu_sets(idx, cnt)


@pytest.mark.parametrize("C,U,kind", [(16, 3, "normal"), (512, 32, "normal"), (1000, 5, "ints"),
                                      (8192, 2, "normal"), (32768, 1, "normal"), (300, 4, "zeros"),
                                      (513, 4, "ints")])
def test_select_topk_exact(csa, C, U, kind):
    """Same fp32 scores on both sides: the sets must agree exactly (ties to
    the lower index, -0 == +0)."""
    if kind == "normal":
        s = _randn((U, C), 8)
    elif kind == "ints":
        s = torch.randint(-3, 4, (U, C), generator=_gen(9), device="cuda").float()
    else:
        s = torch.zeros(U, C, device="cuda")
        s[:, ::3] = -0.0
        s[:, 5::7] = 1.0
    rng = np.random.default_rng(C)
    for k_free, n_sink, n_local in [(2, 1, 1), (29, 1, 2), (0, 1, 1), (C, 0, 0), (C + 5, 2, 3),
                                    (int(rng.integers(1, C)), 0, 1)]:
        got = _run_topk(csa, s, k_free, n_sink, n_local)
        sn = s.cpu().double().numpy()
        for u in range(U):
            ref, _ = O.select_topk(sn[u], k_free, n_sink, n_local)
            assert got[u] == ref, (u, k_free, n_sink, n_local)


@pytest.mark.parametrize("C,U,kind", [(8192, 3, "normal"), (20000, 2, "ints"), (32768, 18, "ints"),
                                      (9000, 4, "zeros")])
def test_select_topk_long_rows_cluster(csa, C, U, kind):
    """Long rows with nothing forced (one cluster per unit, radix select over
    the cluster, ties to the lower index across the CTAs' ranges): the same
    sets as the oracle for k from 0 to past C, many equal scores included."""
    if kind == "normal":
        s = _randn((U, C), 31)
    elif kind == "ints":
        s = torch.randint(-3, 4, (U, C), generator=_gen(32), device="cuda").float()
    else:
        s = torch.zeros(U, C, device="cuda")
        s[:, ::3] = -0.0
        s[:, 5::7] = 1.0
    sn = s.cpu().double().numpy()
    rng = np.random.default_rng(C + U)
    for k_free in [0, 1, 7, C // 3, C - 1, C, C + 5, int(rng.integers(1, C))]:
        got = _run_topk(csa, s, k_free, 0, 0, kmax=C)
        for u in range(U):
            ref, _ = O.select_topk(sn[u], k_free, 0, 0)
            assert got[u] == ref, (u, k_free)


@pytest.mark.parametrize("S,B,Hkv", [(32768, 1, 8), (8192, 2, 3)])
def test_token_select_per_unit_k(csa, S, B, Hkv):
    """csa_token_select: each unit's own k from device memory (0, 1, ties at
    the cut, S) through the cluster path, against the oracle's top-k."""
    U = B * Hkv
    g = _gen(33)
    imp = torch.randint(0, 50, (B, Hkv, S), generator=g, device="cuda").float() / 7.0
    ks = [0, 1, S, S // 2, S - 1] + [int(x) for x in np.random.default_rng(S).integers(1, S, U)]
    k_unit = torch.tensor(ks[:U], dtype=torch.int32, device="cuda")
    idx = torch.full((U, S), 777, dtype=torch.int32, device="cuda")
    cnt = torch.full((U,), 777, dtype=torch.int32, device="cuda")
    csa.csa_token_select(imp, B, S, Hkv, k_unit, idx, cnt)
    csa.csa_check_device_status()
    got = parity.gpu_sets(idx, cnt)
    isn = imp.reshape(U, S).cpu().double().numpy()
    idx_h = idx.cpu().numpy()
    for u in range(U):
        ref, _ = O.select_topk(isn[u], ks[u], 0, 0)
        assert got[u] == ref, (u, ks[u])
        assert np.all(idx_h[u, len(ref):] == -1)


def test_select_topk_n_valid(csa):
    """Causal units: each sees only chunks [0, n_valid) (0, 1, 2 and ragged)."""
    C, U = 515, 40
    s = _randn((U, C), 10)
    nv = [0, 1, 2, 3, 17, 18, 19, 515] + list(np.random.default_rng(1).integers(0, C + 1, U - 8))
    got = _run_topk(csa, s, 16, 1, 1, n_valid=[int(x) for x in nv])
    sn = s.cpu().double().numpy()
    for u in range(U):
        ref, _ = O.select_topk(sn[u], 16, 1, 1, n_valid=int(nv[u]))
        assert got[u] == ref, (u, nv[u])


@pytest.mark.parametrize("tile_m,L,C", [(64, 64, 64), (128, 64, 130), (64, 128, 40), (32, 96, 23)])
def test_select_topk_causal(csa, tile_m, L, C):
    """Query tiles of a causal prefill: tile t sees the chunks that hold a
    key at or before its last row (t + 1) * tile_m - 1; the diagonal chunk is
    the forced local one.  Two (sequence, KV head) rows of tiles."""
    n_tiles = (C * L) // tile_m
    U = 2 * n_tiles
    s = _randn((U, C), 12)
    kmax = min(C, 16 + 2)
    idx = torch.full((U, kmax), 777, dtype=torch.int32, device="cuda")
    cnt = torch.full((U,), 777, dtype=torch.int32, device="cuda")
    csa.csa_select_topk_causal(s, U, C, n_tiles, tile_m, L, 16, 1, 1, idx, cnt, kmax)
    got = parity.gpu_sets(idx, cnt)
    sn = s.cpu().double().numpy()
    for u in range(U):
        last_row = (u % n_tiles + 1) * tile_m - 1
        v = sum(1 for c in range(C) if c * L <= last_row)
        ref, _ = O.select_topk(sn[u], 16, 1, 1, n_valid=v)
        assert got[u] == ref, (u, v)


def test_select_topk_golden(csa):
    for c in pins_golden("topk_cases.json"):
        s = torch.tensor([c["scores"]], dtype=torch.float32, device="cuda")
        nv = None if c["n_valid"] is None else [c["n_valid"]]
        got = _run_topk(csa, s, c["k_free"], c["n_sink"], c["n_local"], n_valid=nv,
                        kmax=len(c["scores"]))
        assert got[0] == c["expect"], c["why"]


def pins_golden(name):
    import pins
    return pins._golden(name)["cases"]


# ---------------------------------------------------------------- top-p

def _run_topp(csa, s, scale, p, budget, n_sink, n_local):
    U, C = s.shape
    kmax = min(C, budget + n_sink + n_local)
    idx = torch.full((U, kmax), 777, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(U, dtype=torch.int32, device="cuda")
    n_p = torch.zeros(U, dtype=torch.int32, device="cuda")
    csa.csa_select_topp(s, U, C, scale, p, budget, n_sink, n_local, idx, cnt, kmax, n_p)
    return parity.gpu_sets(idx, cnt), n_p.cpu().numpy()


def test_select_topp_golden(csa):
    for c in pins_golden("topp_cases.json"):
        s = torch.tensor([c["scores"]], dtype=torch.float32, device="cuda")
        got, n_p = _run_topp(csa, s, c["logit_scale"], c["p"], c["budget"], c["n_sink"],
                             c["n_local"])
        assert got[0] == c["expect"], c["why"]
        if c["n_p"] <= c["budget"]:
            assert n_p[0] == c["n_p"], c["why"]


@pytest.mark.parametrize("C,U,budget,spread", [(1024, 6, 256, 4.0), (1024, 6, 256, 40.0),
                                               (100, 8, 64, 10.0), (2000, 3, 2048, 3.0),
                                               (37, 5, 5, 1.0)])
def test_select_topp_vs_oracle(csa, C, U, budget, spread):
    """Same fp32 scores; the mass cut is fp32 on the GPU and fp64 in the oracle,
    so a mismatch is accepted only at a near-tie (reported)."""
    s = _randn((U, C), 11) * spread
    scale = 1.0 / math.sqrt(128)
    for p in [0.5, 0.9, 0.99]:
        got, n_p = _run_topp(csa, s, scale, p, budget, 1, 2)
        sn = s.cpu().double().numpy()
        refs, gaps = [], []
        for u in range(U):
            r, rn, gap = O.select_topp(sn[u], scale, p, budget, 1, 2)
            refs.append(r)
            gaps.append(gap)
            if rn <= budget and got[u] == r:
                assert n_p[u] == rn
        parity.compare_sets(got, refs, gaps, f"topp C={C} p={p}")


# ---------------------------------------------------------------- hierarchical

@pytest.mark.parametrize("D,C,Gm,top_meta,k_free,G", [(128, 8192, 32, 8, 32, 4),
                                                      (64, 1024, 16, 5, 20, 2),
                                                      (128, 640, 64, 10, 700, 4)])
def test_select_hier_vs_oracle(csa, D, C, Gm, top_meta, k_free, G):
    B, Hkv = 2, 2
    Hq = G * Hkv
    q = _randn((B, Hq, D), 12, torch.bfloat16)
    summ = _randn((B, Hkv, C, D), 13) * 0.1
    meta = torch.empty(B, Hkv, C // Gm, D, device="cuda")
    csa.csa_meta_summaries(summ, B, Hkv, C, D, Gm, meta)
    kmax = min(C, k_free + 3)
    idx = torch.full((B * Hkv, kmax), 777, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B * Hkv, dtype=torch.int32, device="cuda")
    csa.csa_select_hier(q, q.dtype, meta, summ, B, Hq, Hkv, D, C, Gm, top_meta, k_free, 1, 2,
                        idx, cnt, kmax)
    got = parity.gpu_sets(idx, cnt)
    qn, mn, sn = to_np(q), to_np(meta), to_np(summ)
    refs, gaps = [], []
    for b in range(B):
        for h in range(Hkv):
            r, g1, g2 = O.select_hier(qn[b, h * G:(h + 1) * G], mn[b, h], sn[b, h], Gm, top_meta,
                                      k_free, 1, 2)
            refs.append(r)
            gaps.append(min(g1, g2))
    parity.compare_sets(got, refs, gaps, "hier")


@pytest.mark.parametrize("D", [64, 128])
def test_select_hier_golden(csa, D):
    """The hand-worked cases, scalars in the first dimension (D = 128 takes
    the cluster path: the metas and the children split over CTAs)."""
    for c in pins_golden("hier_cases.json"):
        qv = np.array(c["q"], dtype=np.float32)  # [G, 1] scalars
        G = qv.shape[0]
        summ_s = np.array(c["summ"], dtype=np.float32)
        C = len(summ_s)
        q = torch.zeros(1, G, D, device="cuda")
        q[0, :, 0] = torch.tensor(qv[:, 0])
        summ = torch.zeros(1, 1, C, D, device="cuda")
        summ[0, 0, :, 0] = torch.tensor(summ_s)
        meta = torch.empty(1, 1, C // c["Gm"], D, device="cuda")
        csa.csa_meta_summaries(summ, 1, 1, C, D, c["Gm"], meta)
        kmax = C
        idx = torch.full((1, kmax), 777, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        csa.csa_select_hier(q, torch.float32, meta, summ, 1, G, 1, D, C, c["Gm"], c["top_meta"],
                            c["k_free"], c["n_sink"], c["n_local"], idx, cnt, kmax)
        assert parity.gpu_sets(idx, cnt)[0] == c["expect"], c["why"]


# ---------------------------------------------------------------- merge

def test_lse_merge(csa):
    rows, S, D = 37, 20, 128
    o = _randn((rows, S, D), 14)
    lse = _randn((rows, S), 15) * 3
    lse[::2, 5:] = -math.inf
    lse[3, :] = -math.inf  # a row with no tokens at all
    out = torch.empty(rows, D, device="cuda")
    lo = torch.empty(rows, device="cuda")
    csa.csa_lse_merge(o, lse, rows, S, D, out, torch.float32, lo)
    ro, rl = O.lse_merge(to_np(o), to_np(lse))
    assert np.abs(out.cpu().double().numpy() - ro).max() < 1e-5
    got_l = lo.cpu().double().numpy()
    assert np.isneginf(got_l[3]) and np.all(out[3].cpu().numpy() == 0)
    fin = np.isfinite(rl)
    assert np.abs(got_l[fin] - rl[fin]).max() < 1e-5
    outb = torch.empty(rows, D, dtype=torch.bfloat16, device="cuda")
    csa.csa_lse_merge(o, lse, rows, S, D, outb, torch.bfloat16, None)
    assert np.abs(outb.float().cpu().double().numpy() - ro).max() < 2e-2


# ---------------------------------------------------------------- decode

def _decode_case(csa, dtype, B, Hkv, G, D, T, L, sets, full=(), num_parts=0, max_splits=None,
                 seed=16):
    Hq = G * Hkv
    C = T // L
    dt = _dt(dtype)
    q = _randn((B, Hq, D), seed, dt)
    K = _randn((B, Hkv, T, D), seed + 1, dt)
    V = _randn((B, Hkv, T, D), seed + 2, dt)
    U = B * Hkv
    kmax = max(1, max(len(s) for s in sets))
    idx = torch.full((U, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros(U, dtype=torch.int32)
    for u, s in enumerate(sets):
        idx[u, :len(s)] = torch.tensor(sorted(s), dtype=torch.int32)
        cnt[u] = len(s)
    idx, cnt = idx.cuda(), cnt.cuda()
    hf = None
    if full:
        hf = torch.zeros(Hkv, dtype=torch.uint8)
        hf[list(full)] = 1
        hf = hf.cuda()
    P = num_parts or csa.csa_decode_default_parts(dt, D, L)
    S = max_splits or P
    o_part = torch.full((B, Hq, S, D), float("nan"), device="cuda")
    lse_part = torch.full((B, Hq, S), float("nan"), device="cuda")
    scale = 1.0 / math.sqrt(D)
    csa.csa_sparse_decode(q, K, V, dt, idx, cnt, kmax, hf, B, Hq, Hkv, D, T, L, scale, num_parts,
                          S, o_part, lse_part)
    out = torch.empty(B, Hq, D, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    csa.csa_lse_merge(o_part, lse_part, B * Hq, S, D, out, torch.float32, lse)
    csa.csa_check_device_status()
    eff = [list(range(C)) if (u % Hkv) in full else sorted(s) for u, s in enumerate(sets)]
    qn = to_np(q)
    Kc, Vc = K.cpu(), V.cpu()
    # merged output per unit
    for u, s in enumerate(eff):
        b, h = divmod(u, Hkv)
        ro, rl = O.decode_unit(qn[b, h * G:(h + 1) * G], to_np(Kc[b, h]), to_np(Vc[b, h]), s, L,
                               scale)
        got = out[b, h * G:(h + 1) * G].cpu().double().numpy()
        if not s:
            assert np.all(got == 0) and np.all(np.isneginf(lse[b, h * G:(h + 1) * G].cpu().numpy()))
            continue
        parity.assert_close(got, ro, dtype, f"decode unit {u}")
        assert np.abs(lse[b, h * G:(h + 1) * G].cpu().double().numpy() - rl).max() < 1e-3
    # every split partial against the oracle over that split's chunks
    spl = O.decode_partition([len(s) for s in eff], P)
    op, lp = o_part.cpu(), lse_part.cpu()
    for u, s in enumerate(eff):
        b, h = divmod(u, Hkv)
        for slot in range(S):
            rows = slice(h * G, (h + 1) * G)
            if slot < len(spl[u]):
                a0, a1 = spl[u][slot]
                ro, rl = O.decode_unit(qn[b, rows], to_np(Kc[b, h]), to_np(Vc[b, h]), s[a0:a1], L,
                                       scale)
                parity.assert_close(op[b, rows, slot].double().numpy(), ro, dtype,
                                    f"partial u{u} s{slot}")
                assert np.abs(lp[b, rows, slot].double().numpy() - rl).max() < 1e-3
            else:
                assert torch.all(torch.isneginf(lp[b, rows, slot])), (u, slot)


@pytest.mark.parametrize("dtype,D,L,G", [("bf16", 128, 128, 4), ("bf16", 128, 64, 4),
                                         ("bf16", 64, 64, 8), ("bf16", 64, 128, 1),
                                         ("bf16", 128, 64, 2), ("f32", 64, 64, 4),
                                         ("f32", 128, 128, 8)])
def test_sparse_decode_shapes(csa, dtype, D, L, G):
    B, Hkv, C = 2, 3, 24
    rng = np.random.default_rng(D + L + G)
    sets = [sorted(rng.choice(C, size=int(rng.integers(1, 12)), replace=False).tolist())
            for _ in range(B * Hkv)]
    _decode_case(csa, dtype, B, Hkv, G, D, C * L, L, sets, num_parts=13)


def test_sparse_decode_edge_cases(csa):
    # empty unit, single chunk, a full head, more pieces than chunks, one piece
    B, Hkv, G, D, L, C = 1, 4, 4, 128, 64, 9
    sets = [[], [0], [2, 5, 8], [0, 1, 2, 3, 4, 5, 6, 7, 8]]
    _decode_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=40, max_splits=45)
    _decode_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=1)
    _decode_case(csa, "bf16", B, Hkv, G, D, C * L, L, [[3], [0, 8], [], [1]], full=(2,),
                 num_parts=7)
    _decode_case(csa, "f32", B, Hkv, G, 64, C * L, L, sets, num_parts=40, max_splits=45)
    # T == L: one chunk per head
    _decode_case(csa, "bf16", 2, 2, 4, 128, 128, 128, [[0], [0], [], [0]], num_parts=3)


def test_sparse_decode_mixed_heads_default_parts(csa):
    """Full heads (every chunk) and sparse heads in one launch, default grid."""
    B, Hkv, G, D, L, C = 1, 8, 4, 128, 128, 96
    rng = np.random.default_rng(3)
    sets = [sorted(rng.choice(C, size=20, replace=False).tolist()) for _ in range(B * Hkv)]
    _decode_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, full=(0, 1))


def test_device_index_error_reported(csa):
    """An out-of-range chunk index is caught by the kernel's own check (the
    chunk is replaced by chunk 0), reported by csa_check_device_status, and
    the status is cleared afterwards."""
    B, Hkv, G, D, L, C = 1, 1, 4, 128, 64, 4
    q = _randn((B, G, D), 20, torch.bfloat16)
    K = _randn((B, Hkv, C * L, D), 21, torch.bfloat16)
    idx = torch.tensor([[0, 99]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([2], dtype=torch.int32, device="cuda")
    o = torch.empty(B, G, 4, D, device="cuda")
    l = torch.empty(B, G, 4, device="cuda")
    csa.csa_sparse_decode(q, K, K, torch.bfloat16, idx, cnt, 2, None, B, G, Hkv, D, C * L, L, 0.1,
                          4, 4, o, l)
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_check_device_status()
    assert ei.value.status == 5
    csa.csa_check_device_status()  # cleared


def test_bounded_wait_times_out_without_trap(csa):
    """A wait on a barrier nothing arrives on ends as CSA_ERR_TIMEOUT after the
    limit; the context stays usable."""
    csa.csa_selftest_wait_timeout(20_000_000)  # 20 ms
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_check_device_status()
    assert ei.value.status == 4
    csa.csa_check_device_status()
    x = torch.ones(1000, device="cuda")
    assert float(x.sum()) == 1000.0


def test_host_pointer_rejected(csa):
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16)  # host memory
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_sparse_decode(q, q, q, torch.bfloat16, q, q, 1, None, 1, 4, 1, 128, 128, 128, 0.1,
                              1, 1, q, q)
    assert ei.value.status == 1


# ---------------------------------------------------------------- fused paths

@pytest.mark.parametrize("select,R,G,C,ties", [("topk", 0, 4, 512, False), ("topk", 32, 8, 300, False),
                                               ("topk", 0, 4, 4096, False), ("topk", 16, 4, 2048, True),
                                               ("topk", 0, 4, 13, True),
                                               ("topp", 16, 4, 1024, False), ("topp", 0, 2, 700, False)])
def test_fused_score_select_equals_two_calls(csa, select, R, G, C, ties):
    """Scores computed next to the selection (one CTA per unit, or for top-k
    one cluster of CTAs per unit whose best candidates meet in one CTA) give
    the same index lists as csa_score_chunks followed by csa_select_*; with
    integer summaries and queries many scores tie exactly (lower index
    first)."""
    B, Hkv, D = 2, 4, 128
    Hq = G * Hkv
    q = _randn((B, Hq, D), 30, torch.bfloat16)
    P = _randn((D, R), 31) / 4 if R else None
    Ds = R or D
    summ = _randn((B, Hkv, C, Ds), 32) * 0.3
    if ties:
        q = torch.randint(-1, 2, (B, Hq, D), generator=_gen(33), device="cuda").to(torch.bfloat16)
        summ = torch.randint(-1, 2, (B, Hkv, C, Ds), generator=_gen(34), device="cuda").float()
        P = torch.randint(-1, 2, (D, R), generator=_gen(35), device="cuda").float() if R else None
    full = torch.tensor([0, 1, 0, 0], dtype=torch.uint8, device="cuda")
    U = B * Hkv
    kmax = min(C, (20 if select == "topk" else 64) + 3)
    scores = torch.zeros(B, Hkv, 1, C, device="cuda")
    csa.csa_score_chunks(q, q.dtype, P, R, summ, B, 1, Hq, Hkv, D, C, full, 0, 0, scores)
    i1 = torch.full((U, kmax), 7, dtype=torch.int32, device="cuda")
    c1 = torch.zeros(U, dtype=torch.int32, device="cuda")
    i2, c2 = i1.clone(), c1.clone()
    n1 = torch.zeros(U, dtype=torch.int32, device="cuda")
    n2 = n1.clone()
    if select == "topk":
        csa.csa_select_topk(scores, U, C, None, 20, 1, 2, i1, c1, kmax)
        csa.csa_score_select_topk(q, q.dtype, P, R, summ, B, Hq, Hkv, D, C, full, 20, 1, 2, i2, c2,
                                  kmax)
    else:
        for p in (0.9, 0.3):
            csa.csa_select_topp(scores, U, C, D ** -0.5, p, 64, 1, 2, i1, c1, kmax, n1)
            csa.csa_score_select_topp(q, q.dtype, P, R, summ, B, Hq, Hkv, D, C, full, D ** -0.5,
                                      p, 64, 1, 2, i2, c2, kmax, n2)
    for u in range(U):
        if u % Hkv == 1:
            assert int(c2[u]) == 0 and torch.all(i2[u] == -1)
            continue
        assert torch.equal(i1[u], i2[u]) and int(c1[u]) == int(c2[u]), u
        if select == "topp":
            assert int(n1[u]) == int(n2[u])


def _merged_case(csa, dtype, B, Hkv, G, D, T, L, sets, full=(), num_parts=0, out_bf16=False,
                 with_lse=True, seed=40):
    Hq = G * Hkv
    C = T // L
    dt = _dt(dtype)
    q = _randn((B, Hq, D), seed, dt)
    K = _randn((B, Hkv, T, D), seed + 1, dt)
    V = _randn((B, Hkv, T, D), seed + 2, dt)
    U = B * Hkv
    kmax = max(1, max(len(s) for s in sets))
    idx = torch.full((U, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros(U, dtype=torch.int32)
    for u, s in enumerate(sets):
        idx[u, :len(s)] = torch.tensor(sorted(s), dtype=torch.int32)
        cnt[u] = len(s)
    idx, cnt = idx.cuda(), cnt.cuda()
    hf = None
    if full:
        hf = torch.zeros(Hkv, dtype=torch.uint8)
        hf[list(full)] = 1
        hf = hf.cuda()
    scale = D ** -0.5
    nbytes = csa.csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    odt = torch.bfloat16 if out_bf16 else torch.float32
    outs = []
    for _ in range(2):  # the second call must see the counters reset by the first
        out = torch.full((B, Hq, D), float("nan"), device="cuda").to(odt)
        lse = torch.full((B, Hq), float("nan"), device="cuda") if with_lse else None
        csa.csa_sparse_decode_merged(q, K, V, dt, idx, cnt, kmax, hf, B, Hq, Hkv, D, T, L, scale,
                                     num_parts, ws, nbytes, out, odt, lse)
        csa.csa_check_device_status()
        outs.append((out.clone(), None if lse is None else lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert int(ws[:4 * U].view(torch.int32).abs().sum()) == 0  # counters back at zero
    out, lse = outs[1]
    eff = [list(range(C)) if (u % Hkv) in full else sorted(s) for u, s in enumerate(sets)]
    qn = to_np(q)
    Kc, Vc = K.cpu(), V.cpu()
    tol = "bf16" if (dtype == "bf16" or out_bf16) else "f32"
    for u, s in enumerate(eff):
        b, h = divmod(u, Hkv)
        rows = slice(h * G, (h + 1) * G)
        got = out[b, rows].float().cpu().double().numpy()
        if not s:
            assert np.all(got == 0)
            if lse is not None:
                assert torch.all(torch.isneginf(lse[b, rows]))
            continue
        ro, rl = O.decode_unit(qn[b, rows], to_np(Kc[b, h]), to_np(Vc[b, h]), s, L, scale)
        parity.assert_close(got, ro, tol, f"merged unit {u}")
        if lse is not None:
            assert np.abs(lse[b, rows].cpu().double().numpy() - rl).max() < 1e-3
    # same result as the split path (decode + separate merge) with the same
    # pieces, to fp32 rounding (num_parts = 0 lets the library pick a cluster
    # per unit instead: other parts, other bf16 roundings of P, checked
    # against the oracle above)
    if not out_bf16 and num_parts != 0:
        P = num_parts or csa.csa_decode_default_parts(dt, D, L)
        o_part = torch.empty(B, Hq, P, D, device="cuda")
        l_part = torch.empty(B, Hq, P, device="cuda")
        csa.csa_sparse_decode(q, K, V, dt, idx, cnt, kmax, hf, B, Hq, Hkv, D, T, L, scale,
                              num_parts, P, o_part, l_part)
        ref = torch.empty(B, Hq, D, device="cuda")
        csa.csa_lse_merge(o_part, l_part, B * Hq, P, D, ref, torch.float32, None)
        assert (out - ref).abs().max().item() < 1e-5
    return out


@pytest.mark.parametrize("dtype,D,L,G,parts", [("bf16", 128, 128, 4, 0), ("bf16", 128, 64, 4, 13),
                                               ("bf16", 64, 64, 8, 7), ("f32", 64, 64, 4, 5),
                                               ("f32", 128, 128, 2, 0), ("bf16", 64, 128, 1, 256)])
def test_merged_decode_shapes(csa, dtype, D, L, G, parts):
    B, Hkv, C = 2, 3, 24
    rng = np.random.default_rng(D + L + G + parts)
    sets = [sorted(rng.choice(C, size=int(rng.integers(1, 14)), replace=False).tolist())
            for _ in range(B * Hkv)]
    _merged_case(csa, dtype, B, Hkv, G, D, C * L, L, sets, num_parts=parts)


def test_merged_decode_edge_cases(csa):
    B, Hkv, G, D, L, C = 1, 4, 4, 128, 64, 9
    sets = [[], [0], [2, 5, 8], list(range(9))]
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=1)      # one split each
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=200)    # more pieces than chunks
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, [[3], [0, 8], [], [1]], full=(2,), num_parts=7)
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=5, out_bf16=True)
    _merged_case(csa, "f32", B, Hkv, G, 64, C * L, L, sets, num_parts=3, with_lse=False)


@pytest.mark.parametrize("B,Hkv,G,D,L,C,nmax", [(1, 4, 4, 128, 64, 9, 9), (2, 8, 4, 128, 64, 512, 32),
                                                 (1, 8, 4, 128, 128, 300, 35), (3, 2, 8, 64, 64, 40, 20),
                                                 (2, 3, 1, 64, 128, 24, 5), (1, 1, 4, 128, 64, 70, 64),
                                                 (20, 8, 4, 128, 64, 64, 12)])
def test_merged_decode_cluster_path(csa, B, Hkv, G, D, L, C, nmax):
    """Library-chosen pieces (num_parts = 0) on short lists without full
    heads: one cluster of CTAs per unit whose parts meet in distributed
    shared memory (parts of one chunk or none; an empty unit; GQA 1-8; L 64
    and 128).  160 units are more than the SMs: the persistent kernel takes
    them.  Two calls in a row, against the oracle, and against the
    persistent kernel with explicit pieces on the same lists."""
    rng = np.random.default_rng(B * 1000 + Hkv * 100 + C)
    sets = [sorted(rng.choice(C, size=int(rng.integers(1, nmax + 1)), replace=False).tolist())
            for _ in range(B * Hkv)]
    sets[-1] = []  # one unit with no chunk
    out0 = _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=0)
    out1 = _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=148)
    parity.assert_close(out0.cpu().double().numpy(), out1.cpu().double().numpy(), "bf16",
                        "cluster vs persistent")
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=0, out_bf16=True,
                 with_lse=False)


def test_merged_decode_second_wave(csa):
    """More pieces than SMs with long chunk lists: the CTAs of the second wave
    start only when CTAs of the first have retired, and still bring their
    splits to the right units."""
    B, Hkv, G, D, L, C = 2, 4, 4, 128, 64, 400
    rng = np.random.default_rng(11)
    sets = [sorted(rng.choice(C, size=int(rng.integers(150, 400)), replace=False).tolist())
            for _ in range(B * Hkv)]
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, num_parts=256)
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, full=(1,), num_parts=37,
                 out_bf16=True)


def _hybrid_case(csa, B, Hkv, G, D, L, C, sets, full=(), num_parts=0, out_bf16=False,
                 with_lse=True, seed=60, scope="selected"):
    """csa_sparse_decode_merged_hybrid against the oracle's hybrid context:
    random bf16 gist rows (any gist KV is a valid input), every sparse unit
    over its selected chunks' raw KV plus the gist rows of the scope (its
    selected chunks', or every chunk's), full units over their raw chunks
    only."""
    Hq, T = G * Hkv, C * L
    dt = _dt("bf16")
    q = _randn((B, Hq, D), seed, dt)
    K = _randn((B, Hkv, T, D), seed + 1, dt)
    V = _randn((B, Hkv, T, D), seed + 2, dt)
    Kg = _randn((B, Hkv, C, D), seed + 3, dt)
    Vg = _randn((B, Hkv, C, D), seed + 4, dt)
    U = B * Hkv
    kmax = max(1, max(len(s) for s in sets))
    idx = torch.full((U, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros(U, dtype=torch.int32)
    for u, st in enumerate(sets):
        idx[u, :len(st)] = torch.tensor(sorted(st), dtype=torch.int32)
        cnt[u] = len(st)
    idx, cnt = idx.cuda(), cnt.cuda()
    hf = None
    if full:
        hf = torch.zeros(Hkv, dtype=torch.uint8)
        hf[list(full)] = 1
        hf = hf.cuda()
    scale = D ** -0.5
    nbytes = csa.csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    odt = torch.bfloat16 if out_bf16 else torch.float32
    out = torch.full((B, Hq, D), float("nan"), device="cuda").to(odt)
    lse = torch.full((B, Hq), float("nan"), device="cuda") if with_lse else None
    for _ in range(2):  # the second call sees the counters the first left
        csa.csa_sparse_decode_merged_hybrid(q, K, V, Kg, Vg, scope, dt, idx, cnt, kmax, hf, B, Hq,
                                            Hkv, D, T, L, scale, num_parts, ws, nbytes, out, odt,
                                            lse)
        csa.csa_check_device_status()
    qn = to_np(q)
    Kc, Vc, Kgc, Vgc = K.cpu(), V.cpu(), Kg.cpu(), Vg.cpu()
    for u, st in enumerate(sets):
        b, h = divmod(u, Hkv)
        rows = slice(h * G, (h + 1) * G)
        got = out[b, rows].float().cpu().double().numpy()
        if h in full:
            ro, rl = O.decode_unit(qn[b, rows], to_np(Kc[b, h]), to_np(Vc[b, h]), range(C), L,
                                   scale)
        else:
            ro, rl = O.hybrid_unit(qn[b, rows], to_np(Kc[b, h]), to_np(Vc[b, h]),
                                   to_np(Kgc[b, h]), to_np(Vgc[b, h]), st, L, scale, scope)
        parity.assert_close(got, ro, "bf16", f"hybrid {scope} unit {u}")
        if lse is not None:
            gl = lse[b, rows].cpu().double().numpy()
            assert np.array_equal(np.isneginf(gl), np.isneginf(rl)), (u, gl, rl)
            fin = np.isfinite(rl)
            assert np.abs(gl[fin] - rl[fin]).max(initial=0.0) < 1e-3, u
    return out


@pytest.mark.parametrize("scope", ["selected", "all"])
@pytest.mark.parametrize("D,L,G,C,parts", [(128, 128, 4, 24, 0), (128, 64, 4, 150, 13),
                                           (64, 64, 8, 40, 7), (64, 128, 2, 300, 256),
                                           (128, 128, 1, 9, 3)])
def test_hybrid_decode_shapes(csa, D, L, G, C, parts, scope):
    """Gist rows from one ragged chunk (fewer rows than L) to several with a
    ragged last one, GQA groups 1-8, few and many pieces."""
    B, Hkv = 2, 3
    rng = np.random.default_rng(D + L + G + C)
    sets = [sorted(rng.choice(C, size=int(rng.integers(1, min(C, 14) + 1)),
                              replace=False).tolist()) for _ in range(B * Hkv)]
    _hybrid_case(csa, B, Hkv, G, D, L, C, sets, num_parts=parts, scope=scope)


@pytest.mark.parametrize("scope", ["selected", "all"])
def test_hybrid_decode_edge_cases(csa, scope):
    """A unit with no selected chunk: its gist rows alone (scope "all") or an
    empty context, out = 0 and lse = -inf ("selected"); full heads ignore
    the gist rows; bf16 output; one piece; no lse output; more selected
    chunks than one gathered gist chunk holds (L = 64, 80 and 130 chunks)."""
    B, Hkv, G, D, L, C = 1, 4, 4, 128, 64, 9
    sets = [[], [0], [2, 5, 8], list(range(9))]
    _hybrid_case(csa, B, Hkv, G, D, L, C, sets, num_parts=1, scope=scope)
    _hybrid_case(csa, B, Hkv, G, D, L, C, sets, num_parts=200, out_bf16=True, scope=scope)
    _hybrid_case(csa, B, Hkv, G, D, L, C, sets, full=(2,), num_parts=7, with_lse=False,
                 scope=scope)
    _hybrid_case(csa, 2, 8, 4, 128, 128, 96, [list(range(0, 96, 5))] * 16, full=(0, 1),
                 scope=scope)
    rng = np.random.default_rng(5)
    big = [sorted(rng.choice(200, size=n, replace=False).tolist()) for n in (80, 130, 64, 1)]
    _hybrid_case(csa, 1, 4, 4, 128, 64, 200, big, num_parts=0, scope=scope)


def test_hybrid_decode_rejects_fp32_and_unaligned(csa):
    """The hybrid context needs a bf16 cache and 16-byte aligned gist rows;
    a rejected call enqueues nothing."""
    from query_adaptive_chunk_b200.csa import CsaError
    B, Hq, Hkv, D, L, C = 1, 4, 1, 64, 64, 4
    q = torch.zeros(B, Hq, D, device="cuda")
    K = torch.zeros(B, Hkv, C * L, D, device="cuda")
    g = torch.zeros(B, Hkv, C, D, device="cuda")
    idx = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    cnt = torch.ones(1, dtype=torch.int32, device="cuda")
    nbytes = csa.csa_decode_workspace_bytes(B, Hq, Hkv, D, 0)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.zeros(B, Hq, D, device="cuda")
    with pytest.raises(CsaError):
        csa.csa_sparse_decode_merged_hybrid(q, K, K, g, g, "all", torch.float32, idx, cnt, 1, None,
                                            B, Hq, Hkv, D, C * L, L, 0.1, 0, ws, nbytes, out,
                                            torch.float32, None)
    qb, Kb, gb = q.bfloat16(), K.bfloat16(), g.bfloat16()
    with pytest.raises(CsaError):
        csa.csa_sparse_decode_merged_hybrid(qb, Kb, Kb, gb.view(-1)[1:].data_ptr(), gb, "selected",
                                            torch.bfloat16, idx, cnt, 1, None, B, Hq, Hkv, D, C * L,
                                            L, 0.1, 0, ws, nbytes, out, torch.float32, None)
    with pytest.raises(CsaError, match="gist_scope"):
        csa.csa_sparse_decode_merged_hybrid(qb, Kb, Kb, gb, gb, 2, torch.bfloat16, idx, cnt, 1,
                                            None, B, Hq, Hkv, D, C * L, L, 0.1, 0, ws, nbytes, out,
                                            torch.float32, None)


def test_merged_decode_mixed_heads(csa):
    B, Hkv, G, D, L, C = 1, 8, 4, 128, 128, 96
    rng = np.random.default_rng(7)
    sets = [sorted(rng.choice(C, size=20, replace=False).tolist()) for _ in range(B * Hkv)]
    _merged_case(csa, "bf16", B, Hkv, G, D, C * L, L, sets, full=(0, 1))


# ---------------------------------------------------------------- per-head top-k, GQA union

def _union_from_scores(csa, scores, k_free, n_sink, n_local):
    """Run csa_score_select_topk_union on one unit whose per-head scores are
    exactly `scores` [G][C]: one-hot summaries (chunk c = unit vector c) and
    head g's query = its score row, so q_g . summ_c = scores[g][c]."""
    G, C = len(scores), len(scores[0])
    D = 64
    q = torch.zeros(1, G, D, device="cuda")
    q[0, :, :C] = torch.tensor(scores, dtype=torch.float32, device="cuda")
    summ = torch.zeros(1, 1, C, D, device="cuda")
    summ[0, 0, torch.arange(C), torch.arange(C)] = 1.0
    kmax = min(C, G * k_free + n_sink + n_local)
    idx = torch.full((1, max(kmax, 1)), 777, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.csa_score_select_topk_union(q, torch.float32, None, 0, summ, 1, G, 1, D, C, None, k_free,
                                    n_sink, n_local, idx, cnt, max(kmax, 1))
    csa.csa_check_device_status()
    return parity.gpu_sets(idx, cnt)[0]


def test_select_topk_union_golden(csa):
    for c in pins_golden("topk_union_cases.json"):
        got = _union_from_scores(csa, c["scores"], c["k_free"], c["n_sink"], c["n_local"])
        assert got == c["expect"], c["why"]


def test_select_topk_union_random_ties(csa):
    """Integer scores (many exact ties) through the kernel against the oracle."""
    rng = np.random.default_rng(21)
    for trial in range(12):
        G = int(rng.choice([1, 2, 4, 8]))
        C = int(rng.integers(3, 65))
        s = rng.integers(-3, 4, size=(G, C)).astype(np.float64)
        k_free, n_sink, n_local = int(rng.integers(0, C)), int(rng.integers(0, 3)), int(rng.integers(0, 3))
        got = _union_from_scores(csa, s.tolist(), k_free, n_sink, n_local)
        ref, _ = O.select_topk_union(s, k_free, n_sink, n_local)
        assert got == ref, (trial, G, C, k_free)


def test_select_topk_union_single_head_equals_topk(csa):
    """G = 1: the union kernel and the fused top-k give the same lists."""
    B, Hkv, D, C = 2, 3, 128, 777
    q = _randn((B, Hkv, D), 40, torch.bfloat16)
    summ = _randn((B, Hkv, C, D), 41) * 0.3
    kmax = 24 + 3
    outs = []
    for fn in (csa.csa_score_select_topk, csa.csa_score_select_topk_union):
        idx = torch.full((B * Hkv, kmax), 5, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B * Hkv, dtype=torch.int32, device="cuda")
        fn(q, q.dtype, None, 0, summ, B, Hkv, Hkv, D, C, None, 24, 1, 2, idx, cnt, kmax)
        outs.append(parity.gpu_sets(idx, cnt))
    assert outs[0] == outs[1]


def test_select_topk_union_kmax_too_small_rejected(csa):
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_score_select_topk_union(None, torch.bfloat16, None, 0, None, 1, 8, 2, 128, 512,
                                        None, 10, 1, 1, None, None, 20)
    assert ei.value.status == 1 and "kmax" in str(ei.value)


# ---------------------------------------------------------------- RoPE

@pytest.mark.parametrize("dtype,D,period,pos0,theta", [("f32", 128, 4096, 0, 10000.0),
                                                       ("bf16", 128, 131072, 0, 500000.0),
                                                       ("f32", 64, 1, 1048575, 10000.0),
                                                       ("bf16", 64, 7, 123, 100.0)])
def test_rope_matches_oracle(csa, dtype, D, period, pos0, theta):
    """csa_rope against the oracle's fp64 rotation: fp32 to 2e-6 (the angle is
    reduced in double, so positions near 2^20 keep their accuracy); bf16 to
    one rounding of the output."""
    rows = 3 * period if period < 5000 else period
    rows = min(rows, 40000)
    x = _randn((rows, D), 70 + D, _dt(dtype))
    y = torch.empty_like(x)
    csa.csa_rope(x, y, x.dtype, rows, D, period, pos0, theta)
    csa.csa_check_device_status()
    pos = pos0 + np.arange(rows) % period
    ref = O.rope(to_np(x), pos, theta)
    got = y.cpu().double().numpy()
    if dtype == "f32":
        assert np.abs(got - ref).max() < 2e-6
    else:
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
    # in place gives the same bits
    csa.csa_rope(x, x, x.dtype, rows, D, period, pos0, theta)
    assert torch.equal(x, y)


def test_rope_rejects_bad_arguments(csa):
    from query_adaptive_chunk_b200.csa import CsaError
    x = torch.zeros(4, 63, device="cuda")
    with pytest.raises(CsaError):
        csa.csa_rope(x, x, x.dtype, 4, 63, 4, 0, 10000.0)  # odd D
    x = torch.zeros(4, 64, device="cuda")
    with pytest.raises(CsaError):
        csa.csa_rope(x, x, x.dtype, 4, 64, 0, 0, 10000.0)  # period 0
    with pytest.raises(CsaError):
        csa.csa_rope(x, x, x.dtype, 4, 64, 4, 0, 1.0)  # theta must be > 1
