"""The allocation-free merged decode, for callers that cannot allocate device
memory (an application whose own memory pool forbids other allocations, or a
serving loop that must not call cudaMalloc on its hot path).

csa_sparse_decode_merged_noalloc is called through the C ABI and must give
the same output as the workspace entry point, csa_sparse_decode_merged, on
the same inputs, on two calls in a row (the second call finds the scratch
the first one left behind).  This file is named so that pytest collects it
last; it also passes on its own in a fresh process."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _case(B, Hkv, G, D, L, C, full, seed, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    Hq = G * Hkv
    q = torch.randn(B, Hq, D, generator=g, device="cuda").to(dtype)
    K = torch.randn(B, Hkv, C * L, D, generator=g, device="cuda").to(dtype)
    V = torch.randn(B, Hkv, C * L, D, generator=g, device="cuda").to(dtype)
    rng = np.random.default_rng(seed)
    sets = [sorted(rng.choice(C, size=int(rng.integers(0, C // 2)), replace=False).tolist())
            for _ in range(B * Hkv)]
    kmax = max(1, max(len(s) for s in sets))
    idx = torch.full((B * Hkv, kmax), -1, dtype=torch.int32)
    cnt = torch.zeros(B * Hkv, dtype=torch.int32)
    for u, s in enumerate(sets):
        idx[u, :len(s)] = torch.tensor(s, dtype=torch.int32)
        cnt[u] = len(s)
    hf = None
    if full:
        hf = torch.zeros(Hkv, dtype=torch.uint8)
        hf[list(full)] = 1
        hf = hf.cuda()
    return q, K, V, idx.cuda(), cnt.cuda(), kmax, hf


@pytest.mark.parametrize("B,Hkv,G,D,L,C,full,parts,out_dtype", [
    (1, 8, 4, 128, 128, 96, (0, 1), 0, torch.float32),
    (2, 4, 2, 64, 64, 40, (), 37, torch.bfloat16),
])
def test_noalloc_matches_workspace_entry_point(B, Hkv, G, D, L, C, full, parts, out_dtype):
    from query_adaptive_chunk_b200 import csa
    q, K, V, idx, cnt, kmax, hf = _case(B, Hkv, G, D, L, C, full, seed=B * 100 + D)
    Hq, T = G * Hkv, C * L
    scale = 1.0 / math.sqrt(D)
    nbytes = csa.csa_decode_workspace_bytes(B, Hq, Hkv, D, parts)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    ref = torch.empty(B, Hq, D, device="cuda").to(out_dtype)
    ref_lse = torch.empty(B, Hq, device="cuda")
    csa.csa_sparse_decode_merged(q, K, V, q.dtype, idx, cnt, kmax, hf, B, Hq, Hkv, D, T, L, scale,
                                 parts, ws, nbytes, ref, out_dtype, ref_lse)
    csa.csa_check_device_status()
    for _ in range(2):
        out = torch.full((B, Hq, D), float("nan"), device="cuda").to(out_dtype)
        lse = torch.full((B, Hq), float("nan"), device="cuda")
        csa.csa_sparse_decode_merged_noalloc(q, K, V, q.dtype, idx, cnt, kmax, hf, B, Hq, Hkv, D,
                                             T, L, scale, parts, out, out_dtype, lse)
        csa.csa_check_device_status()
        # same tolerance as the merged-vs-split comparison of the other GPU tests
        assert (out.float() - ref.float()).abs().max().item() <= 1e-5
        fin = torch.isfinite(ref_lse)
        assert torch.equal(fin, torch.isfinite(lse))
        assert (lse[fin] - ref_lse[fin]).abs().max().item() <= 1e-5 if fin.any() else True


def test_noalloc_rejects_a_shape_beyond_its_scratch():
    """A shape whose scratch would exceed the built-in area is refused with
    CSA_ERR_UNSUPPORTED before anything is enqueued."""
    from query_adaptive_chunk_b200 import csa
    with pytest.raises(csa.CsaError) as ei:
        csa.csa_sparse_decode_merged_noalloc(None, None, None, torch.bfloat16, None, None, 8, None,
                                             16, 64, 8, 128, 1 << 20, 128, 0.1, 256, None,
                                             torch.float32, None)
    assert ei.value.status == 2
    assert "scratch" in str(ei.value)
