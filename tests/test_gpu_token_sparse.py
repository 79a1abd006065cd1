"""Token Sparse Attention prefill on the GPU against the CPU oracle
(Token Sparse Attention summary, section 2): the proxy importance, the
Dynamic Token Coverage budget, and the whole compress / attend / decompress
pipeline through the C ABI."""
import math

import numpy as np
import pytest
import torch

import parity
from oracle import csa_oracle as O
from oracle.pipeline import to_np

pytestmark = pytest.mark.gpu


def _gen(seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return g


def _inputs(B, S, Hq, Hkv, D, seed):
    g = _gen(seed)
    Q = torch.randn(B, S, Hq, D, generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn(B, Hkv, S, D, generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn(B, Hkv, S, D, generator=g, device="cuda").to(torch.bfloat16)
    return Q, K, V


def _oracle_importance(Q, K, b, h, G, n_obs, scale):
    S = K.shape[2]
    rows = [to_np(Q[b, S - n_obs:, h * G + g]) for g in range(G)]
    pos = np.concatenate([np.arange(S - n_obs, S)] * G)
    return O.token_importance(np.concatenate(rows), to_np(K[b, h]), pos, scale)


# observed rows R = (Hq/Hkv) n_obs: 256 (two 128-row tiles, double-buffered
# accumulators), 128, 512 (single-buffered), 384, 8 (one tile, mostly zero
# padding), 512 with n_obs = 512 (two 256-row copies per head), 48 with
# n_obs = 24 (8-row copies); ragged key blocks (S % 128 != 0) and B > 1
@pytest.mark.parametrize("B,S,Hq,Hkv,D,n_obs", [(1, 2048, 8, 2, 128, 64), (2, 1000, 4, 1, 64, 32),
                                                (1, 4096, 16, 2, 128, 64), (1, 777, 12, 2, 128, 64),
                                                (1, 600, 2, 2, 64, 8), (1, 1536, 2, 2, 128, 512),
                                                (3, 300, 8, 4, 128, 24)])
def test_token_importance_matches_oracle(B, S, Hq, Hkv, D, n_obs):
    from query_adaptive_chunk_b200 import csa
    Q, K, _ = _inputs(B, S, Hq, Hkv, D, seed=S + D)
    G, scale = Hq // Hkv, 1.0 / math.sqrt(D)
    imp = torch.full((B, Hkv, S), float("nan"), device="cuda")
    nb = csa.csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    csa.csa_token_importance(Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp, scratch, nb)
    csa.csa_check_device_status()
    for b in range(B):
        for h in range(Hkv):
            ref = _oracle_importance(Q, K, b, h, G, n_obs, scale)
            got = imp[b, h].cpu().double().numpy()
            assert abs(got.sum() - G * n_obs) < 1e-3 * G * n_obs
            assert np.allclose(got, ref, rtol=1e-3, atol=1e-6), np.abs(got - ref).max()


def test_token_budget_one_cta_per_sequence():
    """More sequences than the SMs hold 8-CTA clusters of (B * 8 > SMs): the
    one-CTA-per-sequence budget kernel, against the oracle's cut."""
    from query_adaptive_chunk_b200 import csa
    B, S, Hkv, tau = 20, 1536, 2, 0.2
    assert B * 8 > torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(11)
    imp_np = (rng.random((B, Hkv, S)) ** 5).astype(np.float32)
    imp = torch.tensor(imp_np, device="cuda")
    k_seq = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    k_unit = torch.full((B * Hkv,), -7, dtype=torch.int32, device="cuda")
    csa.csa_token_budget(imp, B, S, Hkv, tau, 64, k_seq, k_unit)
    csa.csa_check_device_status()
    for b in range(B):
        mass = imp_np[b].astype(np.float64).sum(axis=0)
        ref = O.coverage_budget(mass, tau)
        got = int(k_seq[b])
        if got != ref:
            cum = np.cumsum(np.sort(mass / mass.sum())[::-1])
            top = cum[got - 1] if got > 0 else 0.0
            below = cum[got - 2] if got > 1 else 0.0
            assert top >= (1 - tau) - 1e-6 and below <= (1 - tau) + 1e-6, (b, got, ref)
            parity.NEAR_TIE_LOG.append(("token budget", b, got, ref))
        assert k_unit[b * Hkv:(b + 1) * Hkv].tolist() == [min(S, (got + 63) // 64 * 64)] * Hkv


def test_token_select_one_cta_per_unit():
    """More units than the SMs hold 8-CTA clusters of (B * Hkv * 8 > SMs): the
    one-CTA-per-unit top-k with each unit's k from device memory."""
    from query_adaptive_chunk_b200 import csa
    B, S, Hkv = 5, 8192, 4
    U = B * Hkv
    assert U * 8 > torch.cuda.get_device_properties(0).multi_processor_count
    g = _gen(12)
    imp = torch.randint(0, 40, (B, Hkv, S), generator=g, device="cuda").float() / 9.0
    ks = [0, 1, S, S // 3] + [int(x) for x in np.random.default_rng(13).integers(1, S, U - 4)]
    k_unit = torch.tensor(ks, dtype=torch.int32, device="cuda")
    idx = torch.full((U, S), 777, dtype=torch.int32, device="cuda")
    cnt = torch.full((U,), 777, dtype=torch.int32, device="cuda")
    csa.csa_token_select(imp, B, S, Hkv, k_unit, idx, cnt)
    csa.csa_check_device_status()
    got = parity.gpu_sets(idx, cnt)
    isn = imp.reshape(U, S).cpu().double().numpy()
    for u in range(U):
        ref, _ = O.select_topk(isn[u], ks[u], 0, 0)
        assert got[u] == ref, (u, ks[u])


@pytest.mark.parametrize("S,tau,seed", [(1000, 0.1, 1), (32768, 0.05, 2), (4096, 0.0, 3),
                                        (4096, 0.9, 4), (333, 0.3, 5)])
def test_token_budget_matches_oracle(S, tau, seed):
    """The budget over a seeded importance (heavy-tailed, two heads, some
    exact ties) against the oracle's tail-dropping count; the tile-rounded
    per-unit counts follow."""
    from query_adaptive_chunk_b200 import csa
    rng = np.random.default_rng(seed)
    Hkv = 2
    imp_np = (rng.random((2, Hkv, S)) ** 6).astype(np.float32)
    imp_np[0, :, :10] = imp_np[0, :, 10:20]  # a few equal masses
    imp = torch.tensor(imp_np, device="cuda")
    k_seq = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    k_unit = torch.full((2 * Hkv,), -7, dtype=torch.int32, device="cuda")
    csa.csa_token_budget(imp, 2, S, Hkv, tau, 64, k_seq, k_unit)
    csa.csa_check_device_status()
    for b in range(2):
        mass = imp_np[b].astype(np.float64).sum(axis=0)
        ref = O.coverage_budget(mass, tau)
        got = int(k_seq[b])
        if got != ref:
            # fp32 sums: the cut may move by tokens whose mass is below the
            # rounding of the running sum; the GPU's count must still be a cut
            # of the exact mass curve to within 1e-6 of the total
            cum = np.cumsum(np.sort(mass / mass.sum())[::-1])
            top = cum[got - 1] if got > 0 else 0.0
            below = cum[got - 2] if got > 1 else 0.0
            assert top >= (1 - tau) - 1e-6 and below <= (1 - tau) + 1e-6, (b, got, ref)
            parity.NEAR_TIE_LOG.append(("token budget", b, got, ref))
        kt = min(S, (got + 63) // 64 * 64)
        assert k_unit[b * Hkv:(b + 1) * Hkv].tolist() == [kt] * Hkv


@pytest.mark.parametrize("B,S,Hq,Hkv,n_obs,tau,seed", [(1, 2048, 8, 2, 64, 0.05, 11),
                                                       (2, 1024, 4, 1, 64, 0.2, 12),
                                                       (1, 4096, 8, 2, 32, 0.01, 13)])
def test_token_sparse_prefill_matches_oracle(B, S, Hq, Hkv, n_obs, tau, seed):
    from query_adaptive_chunk_b200 import csa
    D, G = 128, Hq // Hkv
    Q, K, V = _inputs(B, S, Hq, Hkv, D, seed)
    scale = 1.0 / math.sqrt(D)
    nb = csa.csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    Ob = torch.full((B, S, Hq, D), float("nan"), device="cuda").to(torch.bfloat16)
    budget = torch.zeros(B, dtype=torch.int32, device="cuda")
    csa.csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, ws, nb, Ob, budget)
    csa.csa_check_device_status()
    assert not torch.isnan(Ob.float()).any()
    for b in range(B):
        imps = [_oracle_importance(Q, K, b, h, G, n_obs, scale) for h in range(Hkv)]
        k_ref = O.coverage_budget(np.sum(imps, axis=0), tau)
        k_got = int(budget[b])
        cum = np.cumsum(np.sort(np.sum(imps, axis=0) / np.sum(imps))[::-1])
        assert k_got == k_ref or (cum[k_got - 1] >= (1 - tau) - 1e-6 and
                                  (k_got < 2 or cum[k_got - 2] <= (1 - tau) + 1e-6)), (k_got, k_ref)
        kt = min(S, (k_got + 63) // 64 * 64)
        for h in range(Hkv):
            toks = O.select_tokens(imps[h], kt)
            ref = O.token_sparse_head(to_np(Q[b, :, h * G:(h + 1) * G]), to_np(K[b, h]),
                                      to_np(V[b, h]), toks, scale)
            got = Ob[b, :, h * G:(h + 1) * G].float().cpu().double().numpy()
            # rows the GPU kept: nonzero; ambiguous only at importance near-ties
            kept_gpu = np.abs(got).sum(axis=(1, 2)) > 0
            toks = _check_kept_set(kept_gpu, toks, imps[h], kt, S, f"b{b} h{h}")
            if toks is not None:  # near-tie: the oracle over the GPU's own set
                ref = O.token_sparse_head(to_np(Q[b, :, h * G:(h + 1) * G]), to_np(K[b, h]),
                                          to_np(V[b, h]), toks, scale)
            parity.assert_close(got, ref, "bf16", f"token sparse b{b} h{h}")


def _check_kept_set(kept_gpu, toks_ref, imp, kt, S, label):
    """The GPU's kept rows against the oracle's top-kt tokens: identical, or
    different only among tokens whose importance is within 1e-3 (relative)
    of the cut, in which case the GPU's set (of the same size) is returned
    for the oracle to recompute over; None when the sets agree."""
    kept_ref = np.zeros(S, dtype=bool)
    kept_ref[toks_ref] = True
    diff = np.nonzero(kept_gpu != kept_ref)[0]
    if len(diff) == 0:
        return None
    assert int(kept_gpu.sum()) == kt, (label, int(kept_gpu.sum()), kt)
    cut = np.sort(imp)[::-1][kt - 1]
    rel = np.abs(imp[diff] - cut) / cut
    assert rel.max() < 1e-3, (label, diff[:8], rel.max())
    parity.NEAR_TIE_LOG.append(("token sparse set", label, len(diff)))
    print(f"near-tie: token sparse {label}: {len(diff)} tokens swapped at the cut")
    return np.nonzero(kept_gpu)[0].tolist()


def test_token_sparse_prefill_benched_workload():
    """The benched Token Sparse call at full size: the 32K prefill inputs
    (planted chunks), n_obs = 64, tau = 0.1, all 8 KV heads.  The importance
    of every key of every head and the budget against the oracle; per head
    the kept set, a sample of 40 output rows (the first, the last and random
    kept rows, each against the oracle's causal attention over the kept
    tokens) and 16 dropped rows (exactly 0)."""
    from query_adaptive_chunk_b200 import csa, synth
    w = synth.PREFILL_32K
    inp = synth.make_prefill_inputs(w, device="cuda")
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    B, S, Hq, Hkv, D = w.B, w.S, w.Hq, w.Hkv, w.D
    G, n_obs, tau, scale = w.G, 64, 0.1, w.scale
    nb = csa.csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    imp = torch.full((B, Hkv, S), float("nan"), device="cuda")
    csa.csa_token_importance(Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp, scratch, nb)
    nbw = csa.csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs)
    ws = torch.empty(nbw, dtype=torch.uint8, device="cuda")
    Ob = torch.full((B, S, Hq, D), float("nan"), device="cuda").to(torch.bfloat16)
    budget = torch.zeros(B, dtype=torch.int32, device="cuda")
    csa.csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, ws, nbw, Ob, budget)
    csa.csa_check_device_status()
    imps = [_oracle_importance(Q, K, 0, h, G, n_obs, scale) for h in range(Hkv)]
    for h in range(Hkv):
        got = imp[0, h].cpu().double().numpy()
        assert np.allclose(got, imps[h], rtol=1e-3, atol=1e-6), (h, np.abs(got - imps[h]).max())
    mass = np.sum(imps, axis=0)
    k_ref = O.coverage_budget(mass, tau)
    k_got = int(budget[0])
    cum = np.cumsum(np.sort(mass / mass.sum())[::-1])
    assert k_got == k_ref or (cum[k_got - 1] >= (1 - tau) - 1e-6 and
                              (k_got < 2 or cum[k_got - 2] <= (1 - tau) + 1e-6)), (k_got, k_ref)
    kt = min(S, (k_got + 63) // 64 * 64)
    rng = np.random.default_rng(32768)
    Kc, Vc = K[0].cpu(), V[0].cpu()
    for h in range(Hkv):
        got = Ob[0, :, h * G:(h + 1) * G].float().cpu().double().numpy()  # [S, G, D]
        kept_gpu = np.abs(got).sum(axis=(1, 2)) > 0
        toks_ref = O.select_tokens(imps[h], kt)
        toks = _check_kept_set(kept_gpu, toks_ref, imps[h], kt, S, f"h{h}")
        tset = np.asarray(toks if toks is not None else toks_ref, dtype=np.int64)
        picks = np.unique(np.concatenate([[0, kt - 1], rng.choice(kt, size=38, replace=False)]))
        Kh, Vh = to_np(Kc[h][tset]), to_np(Vc[h][tset])
        for i in picks:
            t = int(tset[i])
            qrows = to_np(Q[0, t, h * G:(h + 1) * G])  # [G, D]
            ref = np.stack([O.causal_attend(qrows[g:g + 1], Kh, Vh, tset, t, scale)[0]
                            for g in range(G)])
            parity.assert_close(got[t], ref, "bf16", f"token sparse h{h} row {t}")
        dropped = np.nonzero(~kept_gpu)[0]
        if len(dropped):
            pick = rng.choice(dropped, size=min(16, len(dropped)), replace=False)
            assert np.all(got[pick] == 0), (h, pick)


def _token_steps(csa, Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale):
    """csa_token_importance, _budget, _select, _compress, _attend and
    _decompress called one after the other; returns (O, k_seq)."""
    dev = "cuda"
    U = B * Hkv
    nb = csa.csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs)
    scratch = torch.empty(nb, dtype=torch.uint8, device=dev)
    imp = torch.empty(B, Hkv, S, device=dev)
    csa.csa_token_importance(Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp, scratch, nb)
    k_seq = torch.empty(B, dtype=torch.int32, device=dev)
    k_unit = torch.empty(U, dtype=torch.int32, device=dev)
    csa.csa_token_budget(imp, B, S, Hkv, tau, 64, k_seq, k_unit)
    idx = torch.empty(U, S, dtype=torch.int32, device=dev)
    cnt = torch.empty(U, dtype=torch.int32, device=dev)
    csa.csa_token_select(imp, B, S, Hkv, k_unit, idx, cnt)
    Qc = torch.empty(B, S, Hq, D, dtype=torch.bfloat16, device=dev)
    Kc = torch.empty(B, Hkv, S, D, dtype=torch.bfloat16, device=dev)
    Vc = torch.empty_like(Kc)
    csa.csa_token_compress(Q, K, V, idx, cnt, B, S, Hq, Hkv, D, Qc, Kc, Vc)
    Oc = torch.empty(B, S, Hq, D, dtype=torch.bfloat16, device=dev)
    csa.csa_token_attend(Qc, Kc, Vc, k_unit, B, S, Hq, Hkv, D, scale, Oc)
    nd = csa.csa_token_decompress_scratch_bytes(B, S, Hkv)
    sd = torch.empty(nd, dtype=torch.uint8, device=dev)
    O = torch.full((B, S, Hq, D), float("nan"), device=dev).to(torch.bfloat16)
    csa.csa_token_decompress(Oc, idx, cnt, B, S, Hq, Hkv, D, sd, nd, O)
    return O, k_seq


def test_token_sparse_steps_match_whole_call_and_graph():
    """The separate step calls give the whole call's output bit for bit (two
    sequences with different budgets), and the whole call captured in a CUDA
    graph replays to the same output: the call never reads the budget back
    on the host."""
    from query_adaptive_chunk_b200 import csa
    B, S, Hq, Hkv, D, n_obs, tau = 2, 2048, 8, 2, 128, 64, 0.05
    Q, K, V = _inputs(B, S, Hq, Hkv, D, seed=77)
    Q[1, :, :, :] *= 4  # sharper attention in sequence 1: a different budget
    scale = 1.0 / math.sqrt(D)
    nbw = csa.csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs)
    ws = torch.empty(nbw, dtype=torch.uint8, device="cuda")
    O1 = torch.full((B, S, Hq, D), float("nan"), device="cuda").to(torch.bfloat16)
    bud = torch.zeros(B, dtype=torch.int32, device="cuda")
    csa.csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, ws, nbw, O1, bud)
    O2, k_seq = _token_steps(csa, Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale)
    csa.csa_check_device_status()
    assert torch.equal(bud, k_seq) and bud[0] != bud[1], (bud, k_seq)
    assert torch.equal(O1, O2)
    O3 = torch.full_like(O1, float("nan"))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        csa.csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, ws, nbw, O3,
                                     bud)
    g.replay()
    torch.cuda.synchronize()
    csa.csa_check_device_status()
    assert torch.equal(O1, O3)
    del g


@pytest.mark.parametrize("wname", ["TOKEN_SPARSE_HEAVY_32K", "TOKEN_SPARSE_HEAVY_128K"])
def test_token_sparse_heavy_workload(wname):
    """The high-sparsity workloads at full size (32K and 128K, 20% heavy-hitter
    tokens shared by the KV heads, n_obs = 64, tau = 0.1): the budget keeps a
    small part of the sequence; importance, budget, kept sets and a sample of
    output rows per head against the oracle (as for the benched 32K call).
    At 128K the budget and the token choice run on their cluster paths."""
    from query_adaptive_chunk_b200 import csa, synth
    w = getattr(synth, wname)
    inp = synth.make_prefill_inputs(w, device="cuda")
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    B, S, Hq, Hkv, D = w.B, w.S, w.Hq, w.Hkv, w.D
    G, n_obs, tau, scale = w.G, 64, 0.1, w.scale
    O_gpu, k_seq = _token_steps(csa, Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale)
    csa.csa_check_device_status()
    imps = [_oracle_importance(Q, K, 0, h, G, n_obs, scale) for h in range(Hkv)]
    mass = np.sum(imps, axis=0)
    k_ref = O.coverage_budget(mass, tau)
    k_got = int(k_seq[0])
    cum = np.cumsum(np.sort(mass / mass.sum())[::-1])
    assert k_got == k_ref or (cum[k_got - 1] >= (1 - tau) - 1e-6 and
                              (k_got < 2 or cum[k_got - 2] <= (1 - tau) + 1e-6)), (k_got, k_ref)
    assert k_got <= 0.25 * S, k_got
    kt = min(S, (k_got + 63) // 64 * 64)
    rng = np.random.default_rng(9)
    Kc, Vc = K[0].cpu(), V[0].cpu()
    for h in range(Hkv):
        got = O_gpu[0, :, h * G:(h + 1) * G].float().cpu().double().numpy()
        kept_gpu = np.abs(got).sum(axis=(1, 2)) > 0
        toks_ref = O.select_tokens(imps[h], kt)
        toks = _check_kept_set(kept_gpu, toks_ref, imps[h], kt, S, f"heavy h{h}")
        tset = np.asarray(toks if toks is not None else toks_ref, dtype=np.int64)
        picks = np.unique(np.concatenate([[0, kt - 1], rng.choice(kt, size=30, replace=False)]))
        Kh, Vh = to_np(Kc[h][tset]), to_np(Vc[h][tset])
        for i in picks:
            t = int(tset[i])
            qrows = to_np(Q[0, t, h * G:(h + 1) * G])
            ref = np.stack([O.causal_attend(qrows[g:g + 1], Kh, Vh, tset, t, scale)[0]
                            for g in range(G)])
            parity.assert_close(got[t], ref, "bf16", f"heavy h{h} row {t}")
        dropped = np.nonzero(~kept_gpu)[0]
        pick = rng.choice(dropped, size=min(16, len(dropped)), replace=False)
        assert np.all(got[pick] == 0), (h, pick)


def test_token_sparse_long_batch_on_the_cluster_paths():
    """Two sequences of 65536 tokens (beyond 32768: the budget and the token
    choice on their cluster paths, one cluster per sequence and per KV head),
    with different budgets: budget, kept sets and sampled rows against the
    oracle, dropped rows exactly 0."""
    from query_adaptive_chunk_b200 import csa
    B, S, Hq, Hkv, D, n_obs, tau = 2, 65536, 8, 2, 128, 64, 0.1
    Q, K, V = _inputs(B, S, Hq, Hkv, D, seed=65)
    Q[1] *= 3  # sharper attention in sequence 1: a different budget
    G, scale = Hq // Hkv, 1.0 / math.sqrt(D)
    nbw = csa.csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs)
    ws = torch.empty(nbw, dtype=torch.uint8, device="cuda")
    Ob = torch.full((B, S, Hq, D), float("nan"), device="cuda").to(torch.bfloat16)
    budget = torch.zeros(B, dtype=torch.int32, device="cuda")
    csa.csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, ws, nbw, Ob, budget)
    csa.csa_check_device_status()
    rng = np.random.default_rng(65536)
    for b in range(B):
        imps = [_oracle_importance(Q, K, b, h, G, n_obs, scale) for h in range(Hkv)]
        mass = np.sum(imps, axis=0)
        k_ref = O.coverage_budget(mass, tau)
        k_got = int(budget[b])
        cum = np.cumsum(np.sort(mass / mass.sum())[::-1])
        assert k_got == k_ref or (cum[k_got - 1] >= (1 - tau) - 1e-6 and
                                  (k_got < 2 or cum[k_got - 2] <= (1 - tau) + 1e-6)), (b, k_got, k_ref)
        kt = min(S, (k_got + 63) // 64 * 64)
        Kb, Vb = K[b].cpu(), V[b].cpu()
        for h in range(Hkv):
            got = Ob[b, :, h * G:(h + 1) * G].float().cpu().double().numpy()
            kept_gpu = np.abs(got).sum(axis=(1, 2)) > 0
            toks_ref = O.select_tokens(imps[h], kt)
            toks = _check_kept_set(kept_gpu, toks_ref, imps[h], kt, S, f"long b{b} h{h}")
            tset = np.asarray(toks if toks is not None else toks_ref, dtype=np.int64)
            picks = np.unique(np.concatenate([[0, kt - 1], rng.choice(kt, size=14, replace=False)]))
            Kh, Vh = to_np(Kb[h][tset]), to_np(Vb[h][tset])
            for i in picks:
                t = int(tset[i])
                qrows = to_np(Q[b, t, h * G:(h + 1) * G])
                ref = np.stack([O.causal_attend(qrows[g:g + 1], Kh, Vh, tset, t, scale)[0]
                                for g in range(G)])
                parity.assert_close(got[t], ref, "bf16", f"long b{b} h{h} row {t}")
            dropped = np.nonzero(~kept_gpu)[0]
            if len(dropped):
                pick = rng.choice(dropped, size=min(16, len(dropped)), replace=False)
                assert np.all(got[pick] == 0), (b, h, pick)
    assert int(budget[0]) != int(budget[1]), budget


def test_token_sparse_long_sequences_need_the_cluster_paths():
    """Beyond 32768 tokens the budget and the token choice hold S / 8 values
    per CTA of their cluster paths: with more sequences than the SMs hold
    8-CTA clusters for, the calls are refused (CSA_ERR_UNSUPPORTED) before
    anything is enqueued; above 131072 tokens always."""
    from query_adaptive_chunk_b200 import csa
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, Hkv, S = sms // 8 + 1, 1, 65536
    imp = torch.zeros(B, Hkv, S, device="cuda")
    k_seq = torch.zeros(B, dtype=torch.int32, device="cuda")
    k_unit = torch.zeros(B * Hkv, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_token_budget(imp, B, S, Hkv, 0.1, 64, k_seq, k_unit)
    assert ei.value.status == 2
    idx = torch.zeros(B * Hkv, S, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B * Hkv, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_token_select(imp, B, S, Hkv, k_unit, idx, cnt)
    assert ei.value.status == 2
    imp1 = torch.zeros(1, 1, 2 * 131072, device="cuda")
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_token_budget(imp1, 1, 2 * 131072, 1, 0.1, 64, k_seq[:1], k_unit[:1])
    assert ei.value.status == 2
