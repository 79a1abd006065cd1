"""Whole decode steps through the C ABI (summaries -> score -> select ->
sparse split-K decode -> LSE merge) against the oracle's independent chain
on the same seeded inputs: reduced sizes first, then the full workload sizes
(every unit where the oracle finishes in seconds, sampled units at 1M)."""
import numpy as np
import pytest
import torch

import parity
from oracle import csa_oracle as O
from oracle import pipeline as OP
from oracle.pipeline import to_np
from query_adaptive_chunk_b200 import synth

pytestmark = pytest.mark.gpu


def _decoder(w, inp, fused=True):
    from query_adaptive_chunk_b200.steps import SparseDecoder
    return SparseDecoder(inp["K"], inp["V"], Hq=w.Hq, L=w.L, select=w.select, n_sink=w.n_sink,
                         n_local=w.n_local, k_free=w.k_free, proj=inp.get("proj"), p=w.p,
                         budget=w.budget, full_heads=w.full_heads, Gm=w.Gm, top_meta=w.top_meta,
                         fused=fused, hybrid=w.hybrid,
                         gist=(inp["Kg"], inp["Vg"]) if w.hybrid else None,
                         gist_scope=w.gist_scope or "selected", rope_theta=w.rope_theta)


def run_and_check(w, units=None, fused=True, attention_units=None):
    """One step through the library against the oracle.  Index sets are
    compared on `units` (default: all); outputs on `attention_units`
    (default: the same units)."""
    from query_adaptive_chunk_b200 import csa
    inp = synth.make_decode_inputs(w, device="cuda")
    dec = _decoder(w, inp, fused)
    out, lse = dec.step(inp["q"])
    csa.csa_check_device_status()
    all_units = synth.decode_units(w)
    units = units or all_units
    att = units if attention_units is None else attention_units
    gist = (inp["Kg"], inp["Vg"]) if w.hybrid else None
    kw = dict(L=w.L, scale=w.scale, select=w.select, n_sink=w.n_sink, n_local=w.n_local,
              k_free=w.k_free, proj=inp.get("proj"), p=w.p, budget=w.budget,
              full_heads=w.full_heads, Gm=w.Gm, top_meta=w.top_meta, gist=gist,
              gist_scope=w.gist_scope, rope_theta=w.rope_theta)
    ref = OP.decode_step(inp["q"], inp["K"], inp["V"], units=att, **kw)
    rest = [u for u in units if u not in att]
    if rest:  # index sets only
        r2 = OP.decode_step(inp["q"], inp["K"], inp["V"], units=rest, with_attention=False, **kw)
        for key in ("sets", "gap", "n_p"):
            ref[key].update(r2[key])
    gsets_all = parity.gpu_sets(dec.idx, dec.count)
    sparse = [u for u in units if u[1] not in w.full_heads]
    uidx = {u: i for i, u in enumerate(all_units)}
    n_tie = parity.compare_sets([gsets_all[uidx[u]] for u in sparse],
                                [ref["sets"][u] for u in sparse],
                                [ref["gap"][u] for u in sparse], w.name)
    G = w.G
    worst = 0.0
    for (b, h) in att:
        got = out[b, h * G:(h + 1) * G].cpu().double().numpy()
        gset = list(range(w.C)) if h in w.full_heads else gsets_all[uidx[(b, h)]]
        if gset == ref["sets"][(b, h)]:
            ro, rl = ref["o"][(b, h)], ref["lse"][(b, h)]
        elif w.rope_theta:  # near-tie: rotated attention over the GPU's own set
            tok = O.chunk_tokens(gset, w.L)
            qg = to_np(inp["q"][b, h * G:(h + 1) * G])
            qr = OP._stored(O.rope(qg, np.full(G, OP.rope_query_position(w.T)), w.rope_theta),
                            inp["q"])
            Kr = OP._stored(O.rope(to_np(inp["K"][b, h][tok]), tok, w.rope_theta), inp["K"])
            ro, rl = O.attend(qr, Kr, to_np(inp["V"][b, h][tok]), np.arange(len(tok)), w.scale)
        elif w.hybrid:  # near-tie: the hybrid context over the GPU's own set
            ro, rl = O.hybrid_unit(to_np(inp["q"][b, h * G:(h + 1) * G]), to_np(inp["K"][b, h]),
                                   to_np(inp["V"][b, h]), to_np(inp["Kg"][b, h]),
                                   to_np(inp["Vg"][b, h]), gset, w.L, w.scale, w.gist_scope)
        else:  # near-tie: check attention over the GPU's own set
            ro, rl = O.decode_unit(to_np(inp["q"][b, h * G:(h + 1) * G]), to_np(inp["K"][b, h]),
                                   to_np(inp["V"][b, h]), gset, w.L, w.scale)
        mx, _ = parity.assert_close(got, ro, w.dtype, f"{w.name} unit {(b, h)}")
        worst = max(worst, mx)
        assert np.abs(lse[b, h * G:(h + 1) * G].cpu().double().numpy() - rl).max() < 1e-3
    if w.select == "topp":
        n_p = dec.n_p.cpu().numpy()
        for (b, h) in sparse:
            rn = ref["n_p"][(b, h)]
            if rn <= w.budget:
                assert n_p[uidx[(b, h)]] == rn or ref["gap"][(b, h)] < parity.NEAR_TIE
            else:
                assert n_p[uidx[(b, h)]] == w.budget + 1 or ref["gap"][(b, h)] < parity.NEAR_TIE
    print(f"{w.name}: units {len(units)} (attention {len(att)}) near-ties {n_tie} "
          f"worst max-abs {worst:.3g}")
    return dec, inp


def test_tiny_f32_decode():
    run_and_check(synth.TINY_F32)


def test_topk_decode_reduced():
    run_and_check(synth.TOPK_32K.scaled(B=2, T=8192))


def test_topk_decode_full_size():
    run_and_check(synth.TOPK_32K)


def test_topk_decode_full_size_separate_calls():
    run_and_check(synth.TOPK_32K, fused=False)


def test_topp_decode_prefix_cut():
    """C = 128 < budget: the cap cannot bind, the mass cut p decides."""
    run_and_check(synth.TOPP_128K.scaled(T=16384))


def test_topp_decode_reduced():
    run_and_check(synth.TOPP_128K.scaled(T=65536))


def test_topp_mixed_decode_full_size():
    run_and_check(synth.TOPP_128K)


def test_topp_mixed_decode_full_size_separate_calls():
    run_and_check(synth.TOPP_128K, fused=False)


def test_hier_decode_reduced():
    run_and_check(synth.HIER_1M.scaled(T=131072, planted=8))


def test_topp_mixed_step_batch3_late_merges():
    """The one-call phased step with three sequences (24 units, 6 of them
    full-head): the late CTAs merge the full-head units while the others
    stream the sparse ones; every unit's set and output against the oracle."""
    run_and_check(synth.TOPP_128K.scaled(B=3, T=8192, seed=31))


def test_hier_decode_full_size():
    """1M context: the index sets of all 8 units, the attention of 3."""
    run_and_check(synth.HIER_1M, attention_units=[(0, 0), (0, 5), (0, 7)])


def test_decode_batch_with_gqa8_and_d64():
    w = synth.DecodeWorkload(name="topk_gqa8_d64", seed=11, B=3, Hq=16, Hkv=2, D=64, T=64 * 40,
                             L=64, dtype="bf16", select="topk", n_sink=1, n_local=2, k_free=9,
                             planted=3)
    run_and_check(w)


def test_topk_decode_full_heads_one_call_step():
    """Full and sparse heads in one csa_decode_step: the full heads' chunks
    are decoded while the selection runs, the sparse heads' after it."""
    w = synth.DecodeWorkload(name="topk_mixed_step", seed=12, B=2, Hq=32, Hkv=8, D=128,
                             T=128 * 96, L=128, dtype="bf16", select="topk", n_sink=1, n_local=2,
                             k_free=13, planted=4, full_heads=(0, 3, 7))
    run_and_check(w)


def test_hier_decode_full_heads_one_call_step():
    import dataclasses
    w = dataclasses.replace(synth.HIER_1M.scaled(T=65536, planted=4), name="hier_mixed_step",
                            full_heads=(2,))
    run_and_check(w)


def test_topk_union_decode_reduced():
    """Per-head top-k with the GQA union (each query head's own top-k, the
    group reads the union once)."""
    run_and_check(synth.TOPK_UNION_32K.scaled(B=2, T=8192))


def test_topk_union_decode_full_size():
    run_and_check(synth.TOPK_UNION_32K)


def test_topk_union_with_projection_and_full_head():
    import dataclasses
    w = dataclasses.replace(synth.TOPK_UNION_32K.scaled(B=1, T=16384, planted=4),
                            name="topk_union_proj_mixed", proj_rank=16, full_heads=(3,))
    run_and_check(w)


@pytest.mark.parametrize("w", [synth.HYBRID_TOPK_32K, synth.HYBRID_ALL_TOPK_32K],
                         ids=lambda w: w.gist_scope)
def test_hybrid_topk_decode_reduced(w):
    """SSA's hybrid context through the one-call step: each sparse head over
    the raw KV of its top-k chunks plus gist rows (the chosen chunks' own, or
    every chunk's), the gist rows drawn by the workload generator."""
    run_and_check(w.scaled(B=2, T=8192))


@pytest.mark.parametrize("w", [synth.HYBRID_TOPK_32K, synth.HYBRID_ALL_TOPK_32K],
                         ids=lambda w: w.gist_scope)
def test_hybrid_topk_decode_full_size(w):
    run_and_check(w)


@pytest.mark.parametrize("scope", ["selected", "all"])
def test_hybrid_with_projection_full_head_and_topp(scope):
    """Hybrid context next to a full-attention head, with projected top-p
    scores (the full head attends over its raw tokens only)."""
    import dataclasses
    w = dataclasses.replace(synth.TOPP_128K.scaled(B=1, T=16384), name="hybrid_topp_mixed",
                            seed=17, hybrid=True, gist_scope=scope)
    run_and_check(w)


def test_hybrid_separate_decode_call_matches_step():
    """csa_sparse_decode_merged_hybrid over the step's own index lists gives
    the step's output (same chunk sets, same gist rows)."""
    from query_adaptive_chunk_b200 import csa
    w = synth.HYBRID_TOPK_32K.scaled(B=2, T=8192, planted=2, k_free=100)
    dec, inp = run_and_check(w)
    out_step = dec.out.clone()
    dec.attend(inp["q"])
    csa.csa_check_device_status()
    assert (dec.out - out_step).abs().max().item() < 1e-5


def test_rope_aware_topp_mixed_reduced():
    """RoPE-aware split (RTPurbo review, section 1): chunks scored on the
    pre-RoPE projected keys and query, attention on the rotated cache and
    query (rotated by csa_rope), full and top-p heads in one step."""
    import dataclasses
    w = dataclasses.replace(synth.TOPP_128K.scaled(B=1, T=16384), name="rope_topp_mixed",
                            seed=19, rope_theta=10000.0)
    run_and_check(w)


def test_rope_aware_topk_full_size():
    run_and_check(synth.ROPE_TOPK_32K)


def test_rope_aware_separate_calls_match_step():
    """The separate calls (score on the pre-RoPE query, decode with the
    rotated one) give the one-call step's output."""
    import dataclasses
    from query_adaptive_chunk_b200 import csa
    w = dataclasses.replace(synth.TOPK_32K.scaled(B=2, T=8192), name="rope_topk_small", seed=21,
                            rope_theta=10000.0)
    dec, inp = run_and_check(w)
    out_step = dec.out.clone()
    dec.select_chunks(inp["q"])
    dec.attend(dec.q_rot)
    csa.csa_check_device_status()
    assert (dec.out - out_step).abs().max().item() < 1e-5


def test_decode_step_host_matches_device_step():
    """csa_decode_step_host (query and result in pinned host memory) gives
    the device step's output bit for bit, called directly and replayed as a
    CUDA graph with a new query written into the same host buffer; the
    device step itself is pinned to the oracle by run_and_check."""
    from query_adaptive_chunk_b200 import csa
    w = synth.TOPP_128K.scaled(B=1, T=16384)
    dec, inp = run_and_check(w)
    ref_out, ref_lse = dec.out.clone(), dec.lse.clone()
    q_host = inp["q"].cpu().pin_memory()
    out_host = torch.full(dec.out.shape, float("nan"), dtype=dec.out.dtype).pin_memory()
    lse_host = torch.full(dec.lse.shape, float("nan")).pin_memory()
    dec.step_host(q_host, out_host, lse_host)
    torch.cuda.synchronize()
    csa.csa_check_device_status()
    assert torch.equal(out_host, ref_out.cpu()) and torch.equal(lse_host, ref_lse.cpu())
    # a second query through a graph of the same call
    q2 = (inp["q"].float() * -0.5 + 0.25).to(torch.bfloat16)
    dec.step(q2)
    ref2 = dec.out.clone()
    out_host.fill_(float("nan"))
    g = dec.host_step_graph(q_host, out_host)
    q_host.copy_(q2.cpu())
    out_host.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    csa.csa_check_device_status()
    assert torch.equal(out_host, ref2.cpu())
    del g


def test_decode_step_host_rejects_pageable_and_rope():
    from query_adaptive_chunk_b200 import csa
    w = synth.TOPK_32K.scaled(B=1, T=4096)
    inp = synth.make_decode_inputs(w, device="cuda")
    dec = _decoder(w, inp)
    q_pageable = inp["q"].cpu()
    out_host = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    with pytest.raises(csa.CsaError, match="pinned host memory"):
        dec.step_host(q_pageable, out_host)
    with pytest.raises(csa.CsaError, match="pinned host memory"):
        dec.step_host(inp["q"].cpu().pin_memory(), torch.empty(dec.out.shape))
    dec.desc.q_score = inp["q"].data_ptr()
    with pytest.raises(csa.CsaError, match="CSA_ERR_UNSUPPORTED"):
        csa.csa_decode_step_host(dec.desc, inp["q"].cpu().pin_memory(), out_host)
    dec.desc.q_score = None
    # a selection argument rejected (kmax below the set size) enqueues
    # nothing: the device query buffer keeps what it held
    dec.step_host(inp["q"].cpu().pin_memory(), out_host)
    torch.cuda.synchronize()
    sentinel = torch.full_like(dec.q_dev, 7.0)
    dec.q_dev.copy_(sentinel)
    kmax = dec.desc.kmax
    dec.desc.kmax = 1
    with pytest.raises(csa.CsaError, match="kmax"):
        csa.csa_decode_step_host(dec.desc, (inp["q"] * 0).cpu().pin_memory(), out_host)
    dec.desc.kmax = kmax
    torch.cuda.synchronize()
    assert torch.equal(dec.q_dev, sentinel)
    csa.csa_check_device_status()
