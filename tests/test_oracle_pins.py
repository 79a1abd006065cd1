"""The CPU oracle against its pins (library routines, closed forms, invariants
and hand-enumerated cases); no GPU needed."""
import numpy as np
import pytest
import torch

import pins
from oracle import csa_oracle as O
from oracle import pipeline as P
from query_adaptive_chunk_b200 import synth


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_attention_vs_sdpa_shapes(seed):
    pins.check_attention_vs_sdpa(seed=seed, G=8, D=64, T=1024, L=64, n_sel=4)


def test_planted_chunks_recovered_topk():
    """Sanity (not parity): on a reduced top-k decode workload with uniform
    planting, every planted chunk is selected by the oracle."""
    w = synth.TOPK_32K.scaled(B=2, T=8192)
    inp = synth.make_decode_inputs(w)
    res = P.decode_step(inp["q"], inp["K"], inp["V"], L=w.L, scale=w.scale, select="topk",
                        n_sink=w.n_sink, n_local=w.n_local, k_free=w.k_free,
                        with_attention=False)
    for u, (b, h) in enumerate(synth.decode_units(w)):
        assert set(inp["planted"][u]) <= set(res["sets"][(b, h)])
        assert len(res["sets"][(b, h)]) == w.kmax


def test_planted_chunks_recovered_hier():
    """Sanity: with the hierarchy, a planted chunk whose meta-chunk survives is
    selected."""
    w = synth.HIER_1M.scaled(T=65536, planted=4)
    inp = synth.make_decode_inputs(w)
    res = P.decode_step(inp["q"], inp["K"], inp["V"], L=w.L, scale=w.scale, select="hier",
                        n_sink=w.n_sink, n_local=w.n_local, k_free=w.k_free, Gm=w.Gm,
                        top_meta=w.top_meta, units=[(0, 0), (0, 3)], with_attention=False)
    for (b, h) in [(0, 0), (0, 3)]:
        s = set(res["sets"][(b, h)])
        assert {0, w.C - 2, w.C - 1} <= s and len(s) == 35
        assert set(inp["planted"][h]) <= s


def test_topp_cap_binds_on_zipf_workload():
    """On the Zipf-planted projected workload the prefix mass grows slowly: the
    oracle records n_p > budget on a reduced copy, so the cap decides the set
    (reported, not hidden)."""
    w = synth.TOPP_128K.scaled(T=65536)
    inp = synth.make_decode_inputs(w)
    res = P.decode_step(inp["q"], inp["K"], inp["V"], L=w.L, scale=w.scale, select="topp",
                        n_sink=w.n_sink, n_local=w.n_local, proj=inp["proj"], p=w.p,
                        budget=w.budget, units=[(0, 2), (0, 5)], with_attention=False)
    for u in [(0, 2), (0, 5)]:
        assert res["n_p"][u] >= 1
        assert len(res["sets"][u]) <= w.budget + 3


def test_decode_step_matches_sdpa_on_workload():
    """Whole-step driver: attention output of a unit equals fp64 SDPA masked
    to the unit's chosen chunks (reduced tiny fp32 workload)."""
    w = synth.TINY_F32
    inp = synth.make_decode_inputs(w)
    res = P.decode_step(inp["q"], inp["K"], inp["V"], L=w.L, scale=w.scale, select="topk",
                        n_sink=w.n_sink, n_local=w.n_local, k_free=w.k_free)
    chunks = res["sets"][(0, 0)]
    assert len(chunks) == 4 and {0, 15} <= set(chunks)
    keep = torch.zeros(w.T, dtype=torch.bool)
    for c in chunks:
        keep[c * w.L:(c + 1) * w.L] = True
    q = inp["q"][0].double()[:, None, :]
    K = inp["K"][0, 0].double().expand(w.Hq, -1, -1)
    V = inp["V"][0, 0].double().expand(w.Hq, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None], K[None], V[None], attn_mask=keep.view(1, 1, 1, -1), scale=w.scale)[0, :, 0]
    assert np.allclose(res["o"][(0, 0)], ref.numpy(), rtol=0, atol=1e-12)


def test_prefill_units_dense_small():
    """Prefill driver on a small sequence where every tile keeps all of its
    visible chunks equals causal SDPA."""
    w = synth.PREFILL_32K.scaled(S=512, Hq=8, Hkv=2, k_free=16)
    inp = synth.make_prefill_inputs(w)
    units = [(0, t, h) for t in range(w.n_tiles) for h in range(w.Hkv)]
    res = P.prefill_units(inp["Q"], inp["K"], inp["V"], tile_m=w.tile_m, L=w.L, scale=w.scale,
                          k_free=w.k_free, n_sink=1, n_local=1, units=units)
    Q = inp["Q"][0].double().permute(1, 0, 2)  # [Hq, S, D]
    K = inp["K"][0].double().repeat_interleave(w.G, dim=0)
    V = inp["V"][0].double().repeat_interleave(w.G, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None],
                                                           is_causal=True, scale=w.scale)[0]
    for (b, t, h), o in res["O"].items():
        assert res["sets"][(b, t, h)] == list(range(t + 1))
        want = ref[h * w.G:(h + 1) * w.G, t * w.tile_m:(t + 1) * w.tile_m].numpy()
        assert np.allclose(o, want, rtol=0, atol=1e-12)
