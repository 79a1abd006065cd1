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


@pytest.mark.parametrize("B,S,Hq,Hkv,D,n_obs", [(1, 2048, 8, 2, 128, 64), (2, 1000, 4, 1, 64, 32),
                                                (1, 4096, 16, 2, 128, 64)])
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
            kept_ref = np.zeros(S, dtype=bool)
            kept_ref[toks] = True
            diff = np.nonzero(kept_gpu != kept_ref)[0]
            if len(diff):
                cut = np.sort(imps[h])[::-1][kt - 1]
                rel = np.abs(imps[h][diff] - cut) / cut
                assert rel.max() < 1e-3, (h, diff[:8], rel.max())
                parity.NEAR_TIE_LOG.append(("token sparse set", b, h, len(diff)))
                continue  # outputs of later rows shift with the set: compared where sets agree
            parity.assert_close(got, ref, "bf16", f"token sparse b{b} h{h}")
