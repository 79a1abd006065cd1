"""Block-sparse causal prefill through the C ABI (tcgen05 kernel) against the
oracle: dense-causal special case, sparse chunk unions, hand-built index
lists with empty units, and the full 32K workload on sampled tiles."""
import numpy as np
import pytest
import torch

import parity
from oracle import csa_oracle as O
from oracle import pipeline as OP
from oracle.pipeline import to_np
from query_adaptive_chunk_b200 import synth

pytestmark = pytest.mark.gpu


def _prefill(w, inp):
    from query_adaptive_chunk_b200.steps import BlockSparsePrefill
    return BlockSparsePrefill(inp["Q"], inp["K"], inp["V"], tile_m=w.tile_m, L=w.L,
                              k_free=w.k_free, n_sink=w.n_sink, n_local=w.n_local)


def check(w, units=None):
    from query_adaptive_chunk_b200 import csa
    inp = synth.make_prefill_inputs(w, device="cuda")
    pf = _prefill(w, inp)
    O_gpu = pf.step()
    csa.csa_check_device_status()
    all_units = [(b, h, t) for b in range(w.B) for h in range(w.Hkv) for t in range(w.n_tiles)]
    units = units or [(b, t, h) for (b, h, t) in all_units]
    ref = OP.prefill_units(inp["Q"], inp["K"], inp["V"], tile_m=w.tile_m, L=w.L, scale=w.scale,
                           k_free=w.k_free, n_sink=w.n_sink, n_local=w.n_local, units=units)
    gsets = parity.gpu_sets(pf.idx, pf.count)
    sel_row = lambda b, t, h: (b * w.Hkv + h) * w.n_tiles + t
    n_tie = parity.compare_sets([gsets[sel_row(*u)] for u in units], [ref["sets"][u] for u in units],
                                [ref["gap"][u] for u in units], w.name)
    G = w.G
    Ob = O_gpu.cpu()
    worst = 0.0
    for (b, t, h) in units:
        rows = slice(t * w.tile_m, (t + 1) * w.tile_m)
        got = Ob[b, rows, h * G:(h + 1) * G].permute(1, 0, 2).double().numpy()  # [G, m, D]
        gs = gsets[sel_row(b, t, h)]
        if gs == ref["sets"][(b, t, h)]:
            want = ref["O"][(b, t, h)]
        else:
            want = np.stack([O.prefill_tile(to_np(inp["Q"][b, rows, h * G + g]), to_np(inp["K"][b, h]),
                                            to_np(inp["V"][b, h]), gs, w.L, t * w.tile_m, w.scale)
                             for g in range(G)])
        mx, _ = parity.assert_close(got, want, "bf16", f"{w.name} unit {(b, t, h)}")
        worst = max(worst, mx)
    print(f"{w.name}: units {len(units)} near-ties {n_tie} worst max-abs {worst:.3g}")
    return O_gpu, inp


def test_prefill_dense_causal_small():
    """S = 1024: every tile keeps all its visible chunks, so the prefill is
    plain causal attention (also checked against torch fp64 SDPA)."""
    w = synth.PREFILL_32K.scaled(S=1024)
    O_gpu, inp = check(w)
    Q = inp["Q"][0].double().permute(1, 0, 2).cpu()
    K = inp["K"][0].double().repeat_interleave(w.G, dim=0).cpu()
    V = inp["V"][0].double().repeat_interleave(w.G, dim=0).cpu()
    ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], is_causal=True,
                                                           scale=w.scale)[0]
    got = O_gpu[0].permute(1, 0, 2).cpu().double()
    parity.assert_close(got.numpy(), ref.numpy(), "bf16", "dense causal vs SDPA")


def test_prefill_sparse_medium():
    check(synth.PREFILL_32K.scaled(S=4096))


def test_prefill_batch2_two_kv_heads():
    check(synth.PREFILL_32K.scaled(B=2, S=2048, Hq=8, Hkv=2, planted=3))


def test_prefill_full_size_sampled():
    w = synth.PREFILL_32K
    ts = [0, 1, 2, 16, 17, 18, 100, 255, 256, 400, 510, 511]
    check(w, units=[(0, t, h) for t in ts for h in (0, 3, 7)])


def test_prefill_handbuilt_lists():
    """Index lists given directly: empty units (rows = 0), a single chunk,
    the diagonal alone, and chunks in the middle."""
    from query_adaptive_chunk_b200 import csa
    B, S, Hq, Hkv, D = 1, 512, 8, 2, 128
    n_tiles = S // 64
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    Q = torch.randn(B, S, Hq, D, generator=g, device="cuda").bfloat16()
    K = torch.randn(B, Hkv, S, D, generator=g, device="cuda").bfloat16()
    V = torch.randn(B, Hkv, S, D, generator=g, device="cuda").bfloat16()
    lists = {}
    rng = np.random.default_rng(0)
    for h in range(Hkv):
        for t in range(n_tiles):
            kind = (h * n_tiles + t) % 4
            if kind == 0:
                s = []
            elif kind == 1:
                s = [t]
            elif kind == 2:
                s = [0]
            else:
                s = sorted(set(rng.choice(t + 1, size=min(t + 1, 3), replace=False).tolist()) | {t})
            lists[(h, t)] = s
    kmax = 8
    idx = torch.full((B * Hkv * n_tiles, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros(B * Hkv * n_tiles, dtype=torch.int32)
    for (h, t), s in lists.items():
        r = h * n_tiles + t
        idx[r, :len(s)] = torch.tensor(s, dtype=torch.int32)
        cnt[r] = len(s)
    Og = torch.full((B, S, Hq, D), 7.0, device="cuda").bfloat16()
    csa.csa_block_sparse_prefill(Q, K, V, idx.cuda(), cnt.cuda(), kmax, B, S, Hq, Hkv, D, 64, 64,
                                 D ** -0.5, Og)
    csa.csa_check_device_status()
    G = Hq // Hkv
    for (h, t), s in lists.items():
        rows = slice(t * 64, (t + 1) * 64)
        got = Og[0, rows, h * G:(h + 1) * G].permute(1, 0, 2).cpu().double().numpy()
        want = np.stack([O.prefill_tile(to_np(Q[0, rows, h * G + gg]), to_np(K[0, h]), to_np(V[0, h]),
                                        s, 64, t * 64, D ** -0.5) for gg in range(G)])
        parity.assert_close(got, want, "bf16", f"handbuilt {(h, t)} {s}")


def test_prefill_large_logits_rescale_path():
    """Logits spread over hundreds of units (queries scaled by 8, one chunk
    per KV head with keys scaled by 6): the running row max grows by more
    than 2^8 within a tile, so O is rescaled in tensor memory, and many
    exponentials sit near the bottom of the fp32 range."""
    from query_adaptive_chunk_b200 import csa
    B, S, Hq, Hkv, D = 1, 1024, 8, 2, 128
    n_tiles = S // 64
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    Q = (8 * torch.randn(B, S, Hq, D, generator=g, device="cuda")).bfloat16()
    K = torch.randn(B, Hkv, S, D, generator=g, device="cuda")
    K[:, :, 5 * 64:6 * 64] *= 6
    K = K.bfloat16()
    V = torch.randn(B, Hkv, S, D, generator=g, device="cuda").bfloat16()
    rng = np.random.default_rng(3)
    lists = {}
    for h in range(Hkv):
        for t in range(n_tiles):
            s = set(rng.choice(t + 1, size=min(t + 1, 6), replace=False).tolist()) | {0, t}
            if t > 5:
                s |= {5}
            lists[(h, t)] = sorted(s)
    kmax = 9  # up to 6 random chunks + sink + the large-key chunk + diagonal
    idx = torch.full((B * Hkv * n_tiles, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros(B * Hkv * n_tiles, dtype=torch.int32)
    for (h, t), s in lists.items():
        r = h * n_tiles + t
        idx[r, :len(s)] = torch.tensor(s, dtype=torch.int32)
        cnt[r] = len(s)
    Og = torch.empty(B, S, Hq, D, device="cuda").bfloat16()
    csa.csa_block_sparse_prefill(Q, K, V, idx.cuda(), cnt.cuda(), kmax, B, S, Hq, Hkv, D, 64, 64,
                                 D ** -0.5, Og)
    csa.csa_check_device_status()
    G = Hq // Hkv
    for (h, t), s in lists.items():
        rows = slice(t * 64, (t + 1) * 64)
        got = Og[0, rows, h * G:(h + 1) * G].permute(1, 0, 2).cpu().double().numpy()
        want = np.stack([O.prefill_tile(to_np(Q[0, rows, h * G + gg]), to_np(K[0, h]), to_np(V[0, h]),
                                        s, 64, t * 64, D ** -0.5) for gg in range(G)])
        parity.assert_close(got, want, "bf16", f"large logits {(h, t)} {s}")
