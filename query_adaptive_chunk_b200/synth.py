"""Seeded synthetic workloads for query-adaptive chunk-sparse attention.

This module only draws inputs: queries, keys, values, the 16-dim projection
matrix and the planted "relevant" chunks.  It holds none of the method's
arithmetic (no summaries, scores, selection or attention), so both the CUDA
path and the CPU oracle can take their inputs from it.

Recipe (every tensor from its own torch generator stream, keyed by the
workload's seed and a tensor id: q/Q=0, K=1, V=2, projection=3,
planted-chunk choice=4, Zipf rank permutation=5):

* q, K, V ~ N(0, 1) drawn in fp32.
* Planting: per (sequence b, KV head h) a direction u = normalise(sum of the
  group's query heads), taken in fp64 from the already-rounded queries and
  cast to fp32.  For decode the sum runs over the G query heads of the
  group; for prefill it runs over every position and every head of the
  group.  Chosen chunks get ``+strength * u`` added to every key row, in fp32,
  before keys are rounded to the working dtype.
  - uniform planting: ``planted`` chunks drawn without replacement from the
    index range [n_sink, C - n_local) (prefill: [1, C - 1));
  - Zipf planting: a random permutation ranks the chunks r = 1..C and the
    chunk of rank r gets ``strength * r**(-zipf_s) * u``.
* bf16 workloads round q, K, V to bf16 with round-to-nearest-even after
  planting.
* The projection matrix is N(0, 1) / 4 in fp32, shape [D, R].

Inputs are generated on any torch device; the values depend on the device's
generator, so a test that compares two implementations draws once and hands
the same tensors to both.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "proj": 3, "plant": 4, "perm": 5, "gist_k": 6, "gist_v": 7,
             "heavy_dir": 8, "heavy_pick": 9}


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """One decode step: a single query token per sequence against a KV cache."""

    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    T: int
    L: int
    dtype: str  # "f32" or "bf16"
    select: str  # "topk", "topk_union", "topp" or "hier"
    n_sink: int
    n_local: int
    k_free: int = 0  # top-k / hierarchical: chunks picked besides the forced ones
    planted: int = 0  # uniform planting: chunks per (b, kvh)
    zipf_s: float = 0.0  # > 0: Zipf planting over all chunks
    strength: float = 3.0
    proj_rank: int = 0  # > 0: score on a [D, proj_rank] projection
    p: float = 0.0  # top-p mass target
    budget: int = 0  # top-p cap on the prefix length
    full_heads: tuple = ()  # KV heads that attend to every chunk
    Gm: int = 0  # hierarchical: chunks per meta-chunk
    top_meta: int = 0  # hierarchical: meta-chunks kept
    hybrid: bool = False  # sparse heads also attend over gist rows (one per chunk)
    gist_scope: str = ""  # hybrid: "selected" (the chosen chunks' gist rows) or "all"
    rope_theta: float = 0.0  # > 0: K/q are pre-RoPE; attention on the rotated ones

    @property
    def C(self) -> int:
        return self.T // self.L

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def kmax(self) -> int:
        """Width of one unit's index row: an upper bound on the set size."""
        extra = self.budget if self.select == "topp" else self.k_free
        if self.select == "topk_union":  # one k_free per query head
            extra = self.G * self.k_free
        return min(self.C, extra + self.n_sink + self.n_local)

    @property
    def scale(self) -> float:
        """Attention logit scale 1/sqrt(D) stated with every workload."""
        return 1.0 / math.sqrt(self.D)

    def scaled(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """Block-sparse causal prefill over query tiles."""

    name: str
    seed: int
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    tile_m: int
    L: int
    k_free: int
    n_sink: int = 1
    n_local: int = 1  # the diagonal chunk
    planted: int = 8
    strength: float = 3.0
    dtype: str = "bf16"
    # heavy-hitter tokens: per sequence a seeded fraction of the token
    # positions, shared by its KV heads, whose keys get +heavy_strength * w,
    # with every query row of the group's heads also given +heavy_strength * w
    # (w a seeded random unit direction per (b, kvh)), so that attention mass
    # concentrates on them
    heavy_frac: float = 0.0
    heavy_strength: float = 0.0

    @property
    def C(self) -> int:
        return self.S // self.L

    @property
    def n_tiles(self) -> int:
        return self.S // self.tile_m

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def kmax(self) -> int:
        return min(self.C, self.k_free + self.n_sink + self.n_local)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def scaled(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)


# The five workloads, named for what they are.
TINY_F32 = DecodeWorkload(
    name="tiny_decode_f32_ctx1k", seed=1, B=1, Hq=4, Hkv=1, D=64, T=1024, L=64,
    dtype="f32", select="topk", n_sink=1, n_local=1, k_free=2)
TOPK_32K = DecodeWorkload(
    name="topk_decode_bf16_ctx32k", seed=2, B=4, Hq=32, Hkv=8, D=128, T=32768, L=64,
    dtype="bf16", select="topk", n_sink=1, n_local=2, k_free=29, planted=8)
TOPP_128K = DecodeWorkload(
    name="topp_mixed_decode_bf16_ctx128k", seed=3, B=1, Hq=32, Hkv=8, D=128, T=131072,
    L=128, dtype="bf16", select="topp", n_sink=1, n_local=2, zipf_s=1.2, proj_rank=16,
    p=0.9, budget=256, full_heads=(0, 1))
HIER_1M = DecodeWorkload(
    name="hier_decode_bf16_ctx1m", seed=4, B=1, Hq=32, Hkv=8, D=128, T=1048576, L=128,
    dtype="bf16", select="hier", n_sink=1, n_local=2, k_free=32, planted=16, Gm=32,
    top_meta=8)
PREFILL_32K = PrefillWorkload(
    name="block_sparse_prefill_bf16_seq32k", seed=5, B=1, S=32768, Hq=32, Hkv=8, D=128,
    tile_m=64, L=64, k_free=16)

# Token Sparse Attention in its high-sparsity regime: the 32K prefill shapes
# with 20% heavy-hitter tokens per KV head (keys and queries share a planted
# direction), so the coverage budget keeps a small part of the sequence
TOKEN_SPARSE_HEAVY_32K = dataclasses.replace(
    PREFILL_32K, name="token_sparse_heavy_prefill_bf16_seq32k", seed=9, planted=0,
    heavy_frac=0.2, heavy_strength=8.0)

# The same recipe at the 128K context the Token Sparse page reports its
# speed-up and index overhead at (B=1, Hq=32, Hkv=8, D=128)
TOKEN_SPARSE_HEAVY_128K = dataclasses.replace(
    TOKEN_SPARSE_HEAVY_32K, name="token_sparse_heavy_prefill_bf16_seq128k", seed=10, S=131072)

# Per-head top-k with the GQA union on the 32K shapes: each of the 4 query
# heads of a group keeps its own 29 best chunks, the group reads the union.
TOPK_UNION_32K = dataclasses.replace(TOPK_32K, name="topk_union_decode_bf16_ctx32k", seed=6,
                                     select="topk_union")

# SSA's hybrid context on the 32K top-k step: each sparse head attends over
# the gist and raw KV of its 32 chosen chunks (one extra 64-row chunk of
# gathered gist rows per unit), or, in the "all" scope, over every chunk's
# gist row plus the raw KV of its chunks (8 extra 64-row chunks per unit)
HYBRID_TOPK_32K = dataclasses.replace(TOPK_32K, name="hybrid_topk_decode_bf16_ctx32k", seed=7,
                                      hybrid=True, gist_scope="selected")
HYBRID_ALL_TOPK_32K = dataclasses.replace(TOPK_32K, name="hybrid_all_topk_decode_bf16_ctx32k",
                                          seed=8, hybrid=True, gist_scope="all")

# RTPurbo's RoPE-aware split: the 32K top-k step scored on the pre-RoPE keys
# and query, attending with the rotated ones (base 500000)
ROPE_TOPK_32K = dataclasses.replace(TOPK_32K, name="rope_topk_decode_bf16_ctx32k", seed=20,
                                    rope_theta=500000.0)

DECODE_WORKLOADS = (TINY_F32, TOPK_32K, TOPP_128K, HIER_1M, TOPK_UNION_32K, HYBRID_TOPK_32K,
                    HYBRID_ALL_TOPK_32K, ROPE_TOPK_32K)
ALL_WORKLOADS = DECODE_WORKLOADS + (PREFILL_32K, TOKEN_SPARSE_HEAVY_32K, TOKEN_SPARSE_HEAVY_128K)


def _gen(device, seed: int, tid: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + tid)
    return g


def _randn(shape, device, seed, tid):
    return torch.randn(shape, generator=_gen(device, seed, tid), device=device,
                       dtype=torch.float32)


def _tdtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _unit_dirs(qsum: torch.Tensor) -> torch.Tensor:
    """Normalise rows of a [..., D] fp64 tensor, return fp32."""
    return (qsum / qsum.norm(dim=-1, keepdim=True)).to(torch.float32)


def make_decode_inputs(w: DecodeWorkload, device="cpu") -> dict:
    """Draw q [B,Hq,D], K, V [B,Hkv,T,D] (and proj [D,R]) for a decode workload.

    Returns a dict with the tensors plus ``planted`` (list per (b,kvh) of the
    planted chunk ids, or of the rank permutation for Zipf planting)."""
    dt = _tdtype(w.dtype)
    q = _randn((w.B, w.Hq, w.D), device, w.seed, TENSOR_ID["q"]).to(dt)
    qsum = q.to(torch.float64).view(w.B, w.Hkv, w.G, w.D).sum(dim=2)
    u = _unit_dirs(qsum)  # [B, Hkv, D]
    gk = _gen(device, w.seed, TENSOR_ID["k"])
    gv = _gen(device, w.seed, TENSOR_ID["v"])
    gp = torch.Generator(device="cpu")
    gp.manual_seed(w.seed * 1000 + TENSOR_ID["plant"])
    gperm = torch.Generator(device="cpu")
    gperm.manual_seed(w.seed * 1000 + TENSOR_ID["perm"])
    K = torch.empty((w.B, w.Hkv, w.T, w.D), dtype=dt, device=device)
    V = torch.empty((w.B, w.Hkv, w.T, w.D), dtype=dt, device=device)
    planted = []
    # planted chunks are drawn from the index range between the leading
    # n_sink and the trailing n_local chunks
    free = torch.arange(w.n_sink, max(w.C - w.n_local, w.n_sink), dtype=torch.long)
    for b in range(w.B):
        for h in range(w.Hkv):
            kb = torch.randn((w.T, w.D), generator=gk, device=device, dtype=torch.float32)
            vb = torch.randn((w.T, w.D), generator=gv, device=device, dtype=torch.float32)
            kc = kb.view(w.C, w.L, w.D)
            if w.zipf_s > 0:
                perm = torch.randperm(w.C, generator=gperm)  # perm[r-1] = chunk of rank r
                ranks = torch.empty(w.C, dtype=torch.float64)
                ranks[perm] = torch.arange(1, w.C + 1, dtype=torch.float64)
                amp = (w.strength * ranks.pow(-w.zipf_s)).to(torch.float32).to(device)
                kc += amp.view(w.C, 1, 1) * u[b, h].view(1, 1, w.D)
                planted.append(perm.tolist())
            elif w.planted > 0:
                pick = free[torch.randperm(len(free), generator=gp)[: w.planted]]
                pick = pick.sort().values
                kc[pick.to(device)] += w.strength * u[b, h].view(1, 1, w.D)
                planted.append(pick.tolist())
            else:
                planted.append([])
            K[b, h] = kb.to(dt)
            V[b, h] = vb.to(dt)
    out = {"q": q, "K": K, "V": V, "planted": planted}
    if w.hybrid:
        # gist key / value rows [B, Hkv, C, D]: a trained model's gist KV is an
        # input of the step; drawn here N(0, 1/L), the spread of a mean of L
        # N(0, 1) rows
        shape = (w.B, w.Hkv, w.C, w.D)
        out["Kg"] = (_randn(shape, device, w.seed, TENSOR_ID["gist_k"]) / math.sqrt(w.L)).to(dt)
        out["Vg"] = (_randn(shape, device, w.seed, TENSOR_ID["gist_v"]) / math.sqrt(w.L)).to(dt)
    if w.proj_rank > 0:
        out["proj"] = (_randn((w.D, w.proj_rank), device, w.seed, TENSOR_ID["proj"]) / 4.0)
    return out


def make_prefill_inputs(w: PrefillWorkload, device="cpu") -> dict:
    """Draw Q [B,S,Hq,D], K, V [B,Hkv,S,D] for a prefill workload."""
    dt = _tdtype(w.dtype)
    Q = _randn((w.B, w.S, w.Hq, w.D), device, w.seed, TENSOR_ID["q"]).to(dt)
    qsum = Q.to(torch.float64).view(w.B, w.S, w.Hkv, w.G, w.D).sum(dim=(1, 3))
    u = _unit_dirs(qsum)  # [B, Hkv, D]
    gk = _gen(device, w.seed, TENSOR_ID["k"])
    gv = _gen(device, w.seed, TENSOR_ID["v"])
    gp = torch.Generator(device="cpu")
    gp.manual_seed(w.seed * 1000 + TENSOR_ID["plant"])
    K = torch.empty((w.B, w.Hkv, w.S, w.D), dtype=dt, device=device)
    V = torch.empty((w.B, w.Hkv, w.S, w.D), dtype=dt, device=device)
    free = torch.arange(1, max(w.C - 1, 1), dtype=torch.long)  # never the first or last chunk
    planted = []
    heavy = []
    if w.heavy_frac > 0:
        gdir = torch.Generator(device="cpu")
        gdir.manual_seed(w.seed * 1000 + TENSOR_ID["heavy_dir"])
        ghp = torch.Generator(device="cpu")
        ghp.manual_seed(w.seed * 1000 + TENSOR_ID["heavy_pick"])
        Qf = Q.float()
    for b in range(w.B):
        if w.heavy_frac > 0:
            n_heavy = int(round(w.heavy_frac * w.S))
            pos = torch.randperm(w.S, generator=ghp)[:n_heavy].sort().values
            heavy.append(pos.tolist())
        for h in range(w.Hkv):
            kb = torch.randn((w.S, w.D), generator=gk, device=device, dtype=torch.float32)
            vb = torch.randn((w.S, w.D), generator=gv, device=device, dtype=torch.float32)
            if w.planted > 0 and len(free) > 0:
                pick = free[torch.randperm(len(free), generator=gp)[: w.planted]].sort().values
                kb.view(w.C, w.L, w.D)[pick.to(device)] += w.strength * u[b, h].view(1, 1, w.D)
                planted.append(pick.tolist())
            else:
                planted.append([])
            if w.heavy_frac > 0:
                d = torch.randn(w.D, generator=gdir, dtype=torch.float64)
                d = (d / d.norm()).to(torch.float32).to(device)
                kb[pos.to(device)] += w.heavy_strength * d
                Qf[b, :, h * w.G:(h + 1) * w.G] += w.heavy_strength * d
            K[b, h] = kb.to(dt)
            V[b, h] = vb.to(dt)
    if w.heavy_frac > 0:
        Q = Qf.to(dt)
    return {"Q": Q, "K": K, "V": V, "planted": planted, "heavy": heavy}


def decode_units(w: DecodeWorkload):
    """(b, kvh) pairs in unit order u = b * Hkv + kvh."""
    return [(b, h) for b in range(w.B) for h in range(w.Hkv)]

