"""Decode and prefill steps assembled from the C-ABI calls.

``SparseDecoder`` owns the buffers of one decode configuration (chunk
summaries, scores, index lists, split-K partials, outputs) and runs a step
as: score -> select (top-k / top-p / hierarchical) -> sparse decode ->
LSE merge.  ``BlockSparsePrefill`` runs tile means -> causal scores -> top-k
-> block-sparse prefill.  Buffers come from torch (device memory); every
computation is a call into libcsa.
"""
from __future__ import annotations

import math

import torch

from . import csa


def _dt(t: torch.Tensor) -> int:
    return csa.CSA_BF16 if t.dtype == torch.bfloat16 else csa.CSA_F32


class SparseDecoder:
    """Query-adaptive chunk-sparse decode over a fixed KV cache.

    K, V: [B, Hkv, T, D] (bf16 or fp32, contiguous, on the current device).
    select: "topk" | "topk_union" (per-head top-k, GQA union) | "topp" | "hier".  The summaries (and meta-summaries)
    are computed once here, as part of building the cache.  With fused=True
    (default) a step is two launches: fused score+select (one CTA per unit)
    and the merged split-K decode; fused=False runs the separate calls
    (score, select, decode, merge).  With a bf16 cache and fused=True,
    ``step`` is one call of csa_decode_step, whose decode streams the
    full-attention heads while the selection runs.

    hybrid=True (bf16, fused): every sparse head also attends over gist
    key/value rows (the hybrid context of SSA): those of its selected chunks
    (gist_scope="selected", the method section's reading) or of every chunk
    (gist_scope="all").  gist=(Kg, Vg), each [B, Hkv, T/L, D] bf16, is the
    model's gist KV; when it is not given the rows are built here with the
    cache, as the chunk means of K and V in bf16 (a stand-in).

    rope_theta > 0 (the RoPE-aware split): K and the queries given to ``step``
    are pre-RoPE; chunks are scored on them, and attention runs on rotated
    copies (csa_rope): the cache is rotated once here (positions 0..T-1) and
    each step rotates its query at position T - 1."""

    def __init__(self, K: torch.Tensor, V: torch.Tensor, *, Hq: int, L: int, select: str,
                 n_sink: int, n_local: int, k_free: int = 0, proj: torch.Tensor | None = None,
                 p: float = 0.9, budget: int = 256, full_heads=(), Gm: int = 0, top_meta: int = 0,
                 scale: float | None = None, num_parts: int = 0, out_dtype=torch.float32,
                 fused: bool = True, hybrid: bool = False, gist=None, gist_scope: str = "selected",
                 rope_theta: float = 0.0):
        assert K.is_contiguous() and V.is_contiguous() and K.shape == V.shape
        self.K, self.V = K, V
        B, Hkv, T, D = K.shape
        self.B, self.Hq, self.Hkv, self.T, self.D, self.L = B, Hq, Hkv, T, D, L
        self.C = T // L
        self.select, self.n_sink, self.n_local, self.k_free = select, n_sink, n_local, k_free
        self.p, self.budget, self.Gm, self.top_meta = p, budget, Gm, top_meta
        self.scale = 1.0 / math.sqrt(D) if scale is None else scale
        self.proj = proj
        self.R = 0 if proj is None else proj.shape[1]
        self.dtype = _dt(K)
        dev = K.device
        U = B * Hkv
        Ds = self.R if proj is not None else D
        self.summ = torch.empty(B, Hkv, self.C, Ds, dtype=torch.float32, device=dev)
        csa.csa_chunk_summaries(K, self.dtype, B, Hkv, T, D, L, proj, self.R, self.summ)
        self.meta = None
        if select == "hier":
            self.meta = torch.empty(B, Hkv, self.C // Gm, Ds, dtype=torch.float32, device=dev)
            csa.csa_meta_summaries(self.summ, B, Hkv, self.C, Ds, Gm, self.meta)
        self.rope_theta = float(rope_theta)
        self.K_att, self.q_rot = K, None
        if self.rope_theta > 0:
            assert not hybrid, "the hybrid context is not combined with RoPE here"
            self.K_att = torch.empty_like(K)
            csa.csa_rope(K, self.K_att, self.dtype, B * Hkv * T, D, T, 0, self.rope_theta)
            self.q_rot = torch.empty(B, Hq, D, dtype=K.dtype, device=dev)
        self.Kg = self.Vg = None
        self.gist_scope = gist_scope
        if hybrid and gist is not None:
            assert fused and K.dtype == torch.bfloat16, "the hybrid context needs a fused bf16 decode"
            self.Kg, self.Vg = gist
        elif hybrid:
            assert fused and K.dtype == torch.bfloat16, "the hybrid context needs a fused bf16 decode"
            means = torch.empty(B, Hkv, self.C, D, dtype=torch.float32, device=dev)
            csa.csa_chunk_summaries(K, self.dtype, B, Hkv, T, D, L, None, 0, means)
            self.Kg = means.to(torch.bfloat16)
            csa.csa_chunk_summaries(V, self.dtype, B, Hkv, T, D, L, None, 0, means)
            self.Vg = means.to(torch.bfloat16)
        self.head_full = None
        if full_heads:
            hf = torch.zeros(Hkv, dtype=torch.uint8)
            hf[list(full_heads)] = 1
            self.head_full = hf.to(dev)
        extra = budget if select == "topp" else k_free
        if select == "topk_union":
            extra = (Hq // Hkv) * k_free
        self.kmax = min(self.C, extra + n_sink + n_local)
        self.scores = torch.zeros(B, Hkv, 1, self.C, dtype=torch.float32, device=dev)
        self.idx = torch.full((U, self.kmax), -1, dtype=torch.int32, device=dev)
        self.count = torch.zeros(U, dtype=torch.int32, device=dev)
        self.n_p = torch.zeros(U, dtype=torch.int32, device=dev)
        self.P = num_parts if num_parts > 0 else csa.csa_decode_default_parts(self.dtype, D, L)
        self.max_splits = self.P
        self.o_part = torch.empty(B, Hq, self.max_splits, D, dtype=torch.float32, device=dev)
        self.lse_part = torch.empty(B, Hq, self.max_splits, dtype=torch.float32, device=dev)
        self.out = torch.empty(B, Hq, D, dtype=out_dtype, device=dev)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
        self.fused = fused
        self.num_parts = num_parts
        if fused:
            # sized for the larger of the two P the merged paths may use
            self.ws_bytes = max(csa.csa_decode_workspace_bytes(B, Hq, Hkv, D, self.P),
                                csa.csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts))
            self.workspace = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.desc = None
        self.q_dev = None  # the device query buffer of step_host, made on first use
        if fused and self.dtype == csa.CSA_BF16:
            mode = {"topk": csa.CSA_SELECT_TOPK, "topp": csa.CSA_SELECT_TOPP,
                    "hier": csa.CSA_SELECT_HIER, "topk_union": csa.CSA_SELECT_TOPK_UNION}[select]
            self.desc = csa.decode_step_desc(
                K=self.K_att, V=V, B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, L=L, scale=self.scale,
                head_full=self.head_full, mode=mode, summ=self.summ, proj=proj, R=self.R,
                meta=self.meta, Gm=Gm, top_meta=top_meta, k_free=k_free, n_sink=n_sink,
                n_local=n_local, logit_scale=1.0 / math.sqrt(D), p=p, budget=budget, idx=self.idx,
                count=self.count, kmax=self.kmax, n_p_out=self.n_p, num_parts=num_parts,
                workspace=self.workspace, workspace_bytes=self.ws_bytes, out=self.out,
                out_dtype=self.out.dtype, lse_out=self.lse, Kg=self.Kg, Vg=self.Vg,
                gist_scope=gist_scope)

    def select_chunks(self, q: torch.Tensor, stream=None):
        """Score + select: fills self.idx / self.count (and self.n_p for top-p)."""
        B, Hq, Hkv, D, C = self.B, self.Hq, self.Hkv, self.D, self.C
        U = B * Hkv
        qd = _dt(q)
        if self.select == "hier":
            csa.csa_select_hier(q, qd, self.meta, self.summ, B, Hq, Hkv, D, C, self.Gm,
                                self.top_meta, self.k_free, self.n_sink, self.n_local, self.idx,
                                self.count, self.kmax, stream=stream)
            return
        if self.fused and self.select == "topk":
            csa.csa_score_select_topk(q, qd, self.proj, self.R, self.summ, B, Hq, Hkv, D, C,
                                      self.head_full, self.k_free, self.n_sink, self.n_local,
                                      self.idx, self.count, self.kmax, stream=stream)
            return
        if self.select == "topk_union":  # one call: per-head scores never leave the SM
            csa.csa_score_select_topk_union(q, qd, self.proj, self.R, self.summ, B, Hq, Hkv, D, C,
                                            self.head_full, self.k_free, self.n_sink,
                                            self.n_local, self.idx, self.count, self.kmax,
                                            stream=stream)
            return
        if self.fused and self.select == "topp":
            csa.csa_score_select_topp(q, qd, self.proj, self.R, self.summ, B, Hq, Hkv, D, C,
                                      self.head_full, 1.0 / math.sqrt(D), self.p, self.budget,
                                      self.n_sink, self.n_local, self.idx, self.count, self.kmax,
                                      self.n_p, stream=stream)
            return
        csa.csa_score_chunks(q, qd, self.proj, self.R, self.summ, B, 1, Hq, Hkv, D, C,
                             self.head_full, 0, 0, self.scores, stream=stream)
        if self.select == "topk":
            csa.csa_select_topk(self.scores, U, C, None, self.k_free, self.n_sink, self.n_local,
                                self.idx, self.count, self.kmax, stream=stream)
        elif self.select == "topp":
            csa.csa_select_topp(self.scores, U, C, 1.0 / math.sqrt(D), self.p, self.budget,
                                self.n_sink, self.n_local, self.idx, self.count, self.kmax,
                                self.n_p, stream=stream)
        else:
            raise ValueError(self.select)

    def attend(self, q: torch.Tensor, stream=None):
        """Sparse split-K decode over the current index lists, then the LSE merge
        (one launch when fused)."""
        if self.Kg is not None:
            csa.csa_sparse_decode_merged_hybrid(q, self.K_att, self.V, self.Kg, self.Vg,
                                                self.gist_scope, self.dtype,
                                                self.idx, self.count, self.kmax, self.head_full,
                                                self.B, self.Hq, self.Hkv, self.D, self.T, self.L,
                                                self.scale, self.num_parts, self.workspace,
                                                self.ws_bytes, self.out, _dt(self.out), self.lse,
                                                stream=stream)
            return
        if self.fused:
            csa.csa_sparse_decode_merged(q, self.K_att, self.V, self.dtype, self.idx, self.count,
                                         self.kmax, self.head_full, self.B, self.Hq, self.Hkv,
                                         self.D, self.T, self.L, self.scale, self.num_parts,
                                         self.workspace, self.ws_bytes, self.out, _dt(self.out),
                                         self.lse, stream=stream)
            return
        csa.csa_sparse_decode(q, self.K_att, self.V, self.dtype, self.idx, self.count, self.kmax,
                              self.head_full, self.B, self.Hq, self.Hkv, self.D, self.T, self.L,
                              self.scale, self.P, self.max_splits, self.o_part, self.lse_part,
                              stream=stream)
        csa.csa_lse_merge(self.o_part, self.lse_part, self.B * self.Hq, self.max_splits, self.D,
                          self.out, _dt(self.out), self.lse, stream=stream)

    def step(self, q: torch.Tensor, stream=None):
        qa = q  # the query attention runs with
        if self.q_rot is not None:
            csa.csa_rope(q, self.q_rot, self.dtype, self.B * self.Hq, self.D, 1, self.T - 1,
                         self.rope_theta, stream=stream)
            qa = self.q_rot
        if self.desc is not None and q.dtype == torch.bfloat16:
            self.desc.q = qa.data_ptr()
            self.desc.q_score = q.data_ptr() if self.q_rot is not None else None
            csa.csa_decode_step(self.desc, stream=stream)
            return self.out, self.lse
        self.select_chunks(q, stream)
        self.attend(qa, stream)
        return self.out, self.lse

    def step_host(self, q_host: torch.Tensor, out_host: torch.Tensor,
                  lse_host: torch.Tensor | None = None, stream=None):
        """One step whose query and result live in pinned host memory
        (csa_decode_step_host): q_host [B, Hq, D] bf16 is copied into the
        decoder's own device query buffer, the step runs, and the output
        (and lse, when lse_host is given) are copied into out_host, all
        asynchronously on `stream`: synchronise it before reading out_host.
        Needs the one-call bf16 step without RoPE."""
        if self.desc is None or self.q_rot is not None:
            raise ValueError("step_host needs a fused bf16 decoder without RoPE")
        if self.q_dev is None:
            self.q_dev = torch.empty(self.B, self.Hq, self.D, dtype=torch.bfloat16,
                                     device=self.out.device)
        self.desc.q = self.q_dev.data_ptr()
        self.desc.q_score = None
        csa.csa_decode_step_host(self.desc, q_host, out_host, lse_host, stream=stream)

    def host_step_graph(self, q_host: torch.Tensor, out_host: torch.Tensor,
                        lse_host: torch.Tensor | None = None) -> "torch.cuda.CUDAGraph":
        """``step_host`` on these host buffers captured as a CUDA graph: each
        ``replay()`` copies the current contents of q_host in, runs the step
        and copies the result out (synchronise before reading out_host)."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step_host(q_host, out_host, lse_host)  # warm the capture stream
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            self.step_host(q_host, out_host, lse_host)
        return g


class BlockSparsePrefill:
    """Block-sparse causal prefill: per (tile, KV head) the top-k_free chunks by
    tile-mean score plus the sink and the diagonal chunk."""

    def __init__(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, *, tile_m: int, L: int,
                 k_free: int, n_sink: int = 1, n_local: int = 1, scale: float | None = None):
        B, S, Hq, D = Q.shape
        Hkv = K.shape[1]
        self.Q, self.K, self.V = Q, K, V
        self.B, self.S, self.Hq, self.Hkv, self.D = B, S, Hq, Hkv, D
        self.tile_m, self.L, self.k_free, self.n_sink, self.n_local = tile_m, L, k_free, n_sink, n_local
        self.scale = 1.0 / math.sqrt(D) if scale is None else scale
        self.n_tiles = S // tile_m
        self.C = S // L
        dev = Q.device
        self.kmax = min(self.C, k_free + n_sink + n_local)
        self.summ = torch.empty(B, Hkv, self.C, D, dtype=torch.float32, device=dev)
        csa.csa_chunk_summaries(K, _dt(K), B, Hkv, S, D, L, None, 0, self.summ)
        self.qbar = torch.empty(B, self.n_tiles, Hq, D, dtype=torch.float32, device=dev)
        self.scores = torch.empty(B, Hkv, self.n_tiles, self.C, dtype=torch.float32, device=dev)
        U = B * Hkv * self.n_tiles
        self.idx = torch.full((U, self.kmax), -1, dtype=torch.int32, device=dev)
        self.count = torch.zeros(U, dtype=torch.int32, device=dev)
        self.O = torch.empty(B, S, Hq, D, dtype=torch.bfloat16, device=dev)

    def select_chunks(self, stream=None):
        B, S, Hq, Hkv, D = self.B, self.S, self.Hq, self.Hkv, self.D
        csa.csa_tile_mean_q(self.Q, _dt(self.Q), B, S, Hq, D, self.tile_m, self.qbar, stream=stream)
        csa.csa_score_chunks(self.qbar, csa.CSA_F32, None, 0, self.summ, B, self.n_tiles, Hq, Hkv,
                             D, self.C, None, self.tile_m, self.L, self.scores, stream=stream)
        csa.csa_select_topk_causal(self.scores, B * Hkv * self.n_tiles, self.C, self.n_tiles,
                                   self.tile_m, self.L, self.k_free, self.n_sink, self.n_local,
                                   self.idx, self.count, self.kmax, stream=stream)

    def attend(self, stream=None):
        csa.csa_block_sparse_prefill(self.Q, self.K, self.V, self.idx, self.count, self.kmax,
                                     self.B, self.S, self.Hq, self.Hkv, self.D, self.tile_m,
                                     self.L, self.scale, self.O, stream=stream)

    def step(self, stream=None):
        self.select_chunks(stream)
        self.attend(stream)
        return self.O
