"""Benchmark of query-adaptive chunk-sparse attention on B200.

Headline: one decode step (score -> top-p select -> mixed full/sparse split-K
decode -> LSE merge) on the 128K-token workload (B=1, 32 query / 8 KV heads,
D=128, chunks of 128, top-p 0.9 capped at 256 chunks, KV heads 0-1 full),
reported as µs/step (device time, CUDA events, CUDA-graph replay, L2 flushed
between steps) with the HBM GB/s of the step and a roofline entry for the
decode kernel.  The other workloads (top-k 32K, hierarchical 1M, tiny fp32,
block-sparse prefill 32K in TFLOP/s) ride along under "workloads".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs its own replica (units shard across ranks with no collective on the data
path) and rank 0 prints the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from query_adaptive_chunk_b200 import synth  # noqa: E402

METRIC = "sparse-decode µs/step + HBM GB/s (% of peak) at 128K ctx; prefill TFLOP/s"
HEADLINE = synth.TOPP_128K
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def dist_max(x: float, world: int, device) -> float:
    """Max of a float over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_sum(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_workload(w, rank: int):
    """Each rank draws its own replica of the workload (weak scaling)."""
    return w.scaled(seed=w.seed + 100 * rank) if rank else w


# ---------------------------------------------------------------- measurement helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = f"/tmp/csa_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def file_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_file: str, name: str):
    """DRAM traffic per launch recorded from an ncu capture, if the kernel
    source has not changed since (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(name)
    if not e or e.get("source_hash") != file_hash(kernel_file):
        return None
    return e.get("bytes_per_launch")


def make_flush(dev):
    """Evict the inputs from L2 between timed steps: write a 256 MB buffer,
    then read another 256 MB buffer so that the dirty lines of the write are
    written back before the next timed step starts (not inside it)."""
    wbuf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    rbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        wbuf.zero_()
        rbuf.sum()

    return flush


def decoder_for(w, inp):
    from query_adaptive_chunk_b200.steps import SparseDecoder
    return SparseDecoder(inp["K"], inp["V"], Hq=w.Hq, L=w.L, select=w.select, n_sink=w.n_sink,
                         n_local=w.n_local, k_free=w.k_free, proj=inp.get("proj"), p=w.p,
                         budget=w.budget, full_heads=w.full_heads, Gm=w.Gm, top_meta=w.top_meta,
                         hybrid=w.hybrid, gist=(inp["Kg"], inp["Vg"]) if w.hybrid else None,
                         gist_scope=w.gist_scope or "selected", rope_theta=w.rope_theta)


def selected_bytes(w, dec) -> tuple:
    """(selected KV bytes, summary bytes) the step must read, from the actual
    index counts (full heads: every chunk; hybrid: plus the gist rows)."""
    cnt = dec.count.cpu().tolist()
    elt = 2 if w.dtype == "bf16" else 4
    n = 0
    for u, c in enumerate(cnt):
        n += w.C if (u % w.Hkv) in w.full_heads else c
    kv = n * w.L * w.D * elt * 2
    U_sparse = sum(1 for u in range(w.B * w.Hkv) if (u % w.Hkv) not in w.full_heads)
    if w.hybrid and w.gist_scope == "all":  # a gist key and value row per chunk
        kv += U_sparse * w.C * w.D * elt * 2
    elif w.hybrid:  # a gist key and value row per selected chunk
        kv += sum(c for u, c in enumerate(cnt) if (u % w.Hkv) not in w.full_heads) * w.D * elt * 2
    if w.select == "hier":
        summ = U_sparse * (w.C // w.Gm + w.top_meta * w.Gm) * w.D * 4
    else:
        Ds = w.proj_rank or w.D
        summ = U_sparse * w.C * Ds * 4
    return kv, summ, n


def _ext_event():
    try:
        return torch.cuda.Event(enable_timing=True, external=True)
    except TypeError:
        return None


def time_decode(w, steps: int, warmup: int, flush, graph: bool = True):
    """Device time of `steps` decode steps (L2 flushed before each).

    Two CUDA graphs are replayed alternately inside the timed loop: G1 is
    the step as a user runs it (one csa_decode_step call: selection, then
    the decode launched behind it with programmatic dependent launch) and
    gives the step time from events recorded around the replay; G2 runs the
    selection and the merged decode as two plain launches with events
    between them and gives the decode kernel's own duration (with the
    overlap of G1 the kernel has no duration of its own).  Without graph
    support the step is timed from direct launches."""
    inp = synth.make_decode_inputs(w, device="cuda")
    dec = decoder_for(w, inp)
    q = inp["q"]
    for _ in range(warmup):
        dec.step(q)
    torch.cuda.synchronize()
    ev = [_ext_event() for _ in range(3)]
    evs = [_ext_event() for _ in range(2)]  # around the step, inside G1
    use_graph = graph and all(e is not None for e in ev + evs)
    if use_graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            dec.step(q)  # warm the side stream
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1, capture_error_mode="relaxed"):
            evs[0].record()
            dec.step(q)
            evs[1].record()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, capture_error_mode="relaxed"):
            ev[0].record()
            dec.select_chunks(q)
            ev[1].record()
            dec.attend(q)
            ev[2].record()
        for _ in range(warmup):
            g1.replay()
            g2.replay()
        torch.cuda.synchronize()
    step_ms, dec_ms, sel_ms, launch_ms = [], [], [], []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if use_graph:
            e0.record()
            g1.replay()
            e1.record()
            flush()
            g2.replay()
            torch.cuda.synchronize()
            step_ms.append(evs[0].elapsed_time(evs[1]))
            launch_ms.append(e0.elapsed_time(e1))
            dec_ms.append(ev[1].elapsed_time(ev[2]))
            sel_ms.append(ev[0].elapsed_time(ev[1]))
        else:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record()
            dec.select_chunks(q)
            e[1].record()
            dec.attend(q)
            e[2].record()
            torch.cuda.synchronize()
            step_ms.append(e[0].elapsed_time(e[2]))
            launch_ms.append(e[0].elapsed_time(e[2]))
            dec_ms.append(e[1].elapsed_time(e[2]))
            sel_ms.append(e[0].elapsed_time(e[1]))
    kv, summ, n_chunks = selected_bytes(w, dec)
    res = {"step_ms": step_ms, "decode_ms": dec_ms, "select_ms": sel_ms,
           "step_with_launch_ms": launch_ms, "kv_bytes": kv,
           "summ_bytes": summ,
           "chunks": n_chunks, "graph": use_graph, "dec": dec, "inp": inp}
    return res


def time_decode_rotating(w, inp, steps: int, warmup: int, copies: int = 8):
    """Step and decode-kernel time with inputs larger than L2 instead of a
    flush: `copies` copies of the K/V cache (as the layers of a model would
    hold) used in rotation.  Per copy the two graphs of time_decode: G1 the
    one-call step (events around it), G2 the selection and the merged decode
    as plain launches (events around the decode).  Each timed iteration
    replays G1 of copy k and G2 of copy k + copies/2, so a copy is read every
    copies/2 iterations, with copies - 1 other steps' reads between.  Returns the
    times (ms) and the bytes of one cache copy."""
    q = inp["q"]
    decs = []
    for i in range(copies):
        sub = dict(inp)
        if i > 0:
            sub["K"], sub["V"] = inp["K"].clone(), inp["V"].clone()
        decs.append(decoder_for(w, sub))
    g_step, g_dec, evs = [], [], []
    side = torch.cuda.Stream()
    for d in decs:
        for _ in range(2):
            d.step(q)
            d.select_chunks(q)
            d.attend(q)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            d.step(q)
            d.select_chunks(q)
            d.attend(q)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        e = [_ext_event() for _ in range(4)]
        if any(x is None for x in e):
            return None
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1, capture_error_mode="relaxed"):
            e[0].record()
            d.step(q)
            e[1].record()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, capture_error_mode="relaxed"):
            d.select_chunks(q)
            e[2].record()
            d.attend(q)
            e[3].record()
        g_step.append(g1)
        g_dec.append(g2)
        evs.append(e)
    half = copies // 2
    for i in range(warmup * copies):
        g_step[i % copies].replay()
        g_dec[(i + half) % copies].replay()
    torch.cuda.synchronize()
    dec_ms, step_ms = [], []
    for i in range(steps):
        k, k2 = i % copies, (i + half) % copies
        g_step[k].replay()
        g_dec[k2].replay()
        torch.cuda.synchronize()
        step_ms.append(evs[k][0].elapsed_time(evs[k][1]))
        dec_ms.append(evs[k2][2].elapsed_time(evs[k2][3]))
    cache_bytes = (inp["K"].numel() + inp["V"].numel()) * inp["K"].element_size()
    del g_step, g_dec, decs
    return {"decode_ms": dec_ms, "step_ms": step_ms, "cache_bytes": cache_bytes}


def time_separate_calls(w, steps: int, warmup: int, flush):
    """The headline step as the separate boundary calls (the unfused path):
    csa_score_chunks, csa_select_topp, csa_sparse_decode (split partials) and
    csa_lse_merge, in one CUDA graph with an event between each pair (L2
    flushed before each replay).  Returns each call's times (ms) and the
    partials' bytes the merge reads."""
    from query_adaptive_chunk_b200 import csa
    from query_adaptive_chunk_b200.steps import SparseDecoder, _dt
    assert w.select == "topp"
    inp = synth.make_decode_inputs(w, device="cuda")
    d = SparseDecoder(inp["K"], inp["V"], Hq=w.Hq, L=w.L, select=w.select, n_sink=w.n_sink,
                      n_local=w.n_local, k_free=w.k_free, proj=inp.get("proj"), p=w.p,
                      budget=w.budget, full_heads=w.full_heads, fused=False)
    q = inp["q"]
    qd = _dt(q)
    B, Hq, Hkv, D, C = d.B, d.Hq, d.Hkv, d.D, d.C
    ev = [_ext_event() for _ in range(7)]
    if any(e is None for e in ev):
        return None

    def calls(with_events, pair=False):
        if with_events:
            ev[0].record()
        csa.csa_score_chunks(q, qd, d.proj, d.R, d.summ, B, 1, Hq, Hkv, D, C, d.head_full, 0, 0,
                             d.scores)
        if with_events:
            ev[1].record()
        csa.csa_select_topp(d.scores, B * Hkv, C, 1.0 / math.sqrt(D), d.p, d.budget, d.n_sink,
                            d.n_local, d.idx, d.count, d.kmax, d.n_p)
        if with_events:
            ev[2].record()
        if pair:
            ev[5].record()
        csa.csa_sparse_decode(q, d.K_att, d.V, d.dtype, d.idx, d.count, d.kmax, d.head_full, B,
                              Hq, Hkv, D, d.T, d.L, d.scale, d.P, d.max_splits, d.o_part,
                              d.lse_part)
        if with_events:
            ev[3].record()
        csa.csa_lse_merge(d.o_part, d.lse_part, B * Hq, d.max_splits, D, d.out, _dt(d.out),
                          d.lse)
        if with_events:
            ev[4].record()
        if pair:
            ev[6].record()

    for _ in range(warmup):
        calls(False)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        calls(False)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        calls(True)
    # the decode and the merge with no event between them (the merge is
    # launched behind the decode with programmatic dependent launch)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, capture_error_mode="relaxed"):
        calls(False, pair=True)
    for _ in range(warmup):
        g.replay()
        g2.replay()
    torch.cuda.synchronize()
    names = ("score", "select", "decode", "merge")
    ms = {k: [] for k in names}
    ms["decode_merge"] = []
    for _ in range(steps):
        flush()
        g.replay()
        torch.cuda.synchronize()
        for i, k in enumerate(names):
            ms[k].append(ev[i].elapsed_time(ev[i + 1]))
        flush()
        g2.replay()
        torch.cuda.synchronize()
        ms["decode_merge"].append(ev[5].elapsed_time(ev[6]))
    csa.csa_check_device_status()
    del g, g2
    part_bytes = (d.o_part.numel() + d.lse_part.numel()) * 4
    return {"ms": ms, "merge_read_bytes": part_bytes, "dec": d}


def time_e2e(w, dec, inp, steps: int, flush):
    """Same step through the public API with the query in pinned host memory
    and the output read back to pinned host memory, every step
    (csa_decode_step_host: the copies are inside the timed region).  Timed
    as a CUDA-graph replay of that call (how a serving loop runs it) and as
    direct per-call launches.  Returns (graph ms list or None, eager ms list,
    h2d bytes, d2h bytes)."""
    q_host = inp["q"].cpu().pin_memory()
    out_host = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    host_api = dec.desc is not None and dec.q_rot is None
    q_dev = torch.empty_like(inp["q"])

    def run():
        if host_api:
            dec.step_host(q_host, out_host)
        else:
            q_dev.copy_(q_host, non_blocking=True)
            dec.step(q_dev)
            out_host.copy_(dec.out, non_blocking=True)

    def timed(fn):
        ms = []
        for _ in range(steps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return ms

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    eager = timed(run)
    graph = None
    if host_api:
        g = dec.host_step_graph(q_host, out_host)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        graph = timed(g.replay)
        del g
    return graph, eager, q_host.numel() * q_host.element_size(), \
        out_host.numel() * out_host.element_size()


def host_cpu_model() -> str:
    """The host CPU's model name (first entry of /proc/cpuinfo), or ""."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def diagonal_blocks(idx: torch.Tensor, n_tiles: int) -> int:
    """Executed diagonal blocks of a block-sparse prefill whose chunk equals
    its tile (tile_m == L): the units u = (b * Hkv + h) * n_tiles + t whose
    index row holds chunk t."""
    t = torch.arange(idx.shape[0], dtype=torch.int64) % n_tiles
    return int((idx.to(torch.int64) == t[:, None]).any(dim=1).sum())


def time_prefill(w, steps: int, warmup: int, flush):
    from query_adaptive_chunk_b200.steps import BlockSparsePrefill
    inp = synth.make_prefill_inputs(w, device="cuda")
    pf = BlockSparsePrefill(inp["Q"], inp["K"], inp["V"], tile_m=w.tile_m, L=w.L, k_free=w.k_free,
                            n_sink=w.n_sink, n_local=w.n_local)
    for _ in range(warmup):
        pf.step()
    torch.cuda.synchronize()
    sel_ms, att_ms = [], []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        pf.select_chunks()
        e[1].record()
        pf.attend()
        e[2].record()
        torch.cuda.synchronize()
        sel_ms.append(e[0].elapsed_time(e[1]))
        att_ms.append(e[1].elapsed_time(e[2]))
    cnt = pf.count.cpu()
    blocks = int(cnt.sum())
    per_block = w.G * 2 * (2 * w.tile_m * w.L * w.D)
    flops = blocks * per_block
    # causal-effective count: a diagonal block does about half the work
    diag = diagonal_blocks(pf.idx.cpu(), pf.n_tiles) if w.tile_m == w.L else 0
    return {"select_ms": sel_ms, "attend_ms": att_ms, "blocks": blocks, "flops": flops,
            "causal_flops": (blocks - diag / 2) * per_block, "diagonal_blocks": diag}


TOKEN_STAGES = ("importance", "budget", "select", "compress", "attend", "decompress")


def time_token_sparse(w, steps: int, warmup: int, flush, n_obs: int = 64, tau: float = 0.1,
                      dense: bool = False):
    """Token Sparse Attention prefill (importance, budget, each KV head's own
    tokens, compress, dense causal attention of the kept tokens, decompress).

    Two CUDA graphs replayed alternately, L2 flushed before each: G1 is the
    whole call (csa_token_sparse_prefill) between events and gives the
    per-call time; G2 runs the same six steps as the separate calls with an
    event between each pair and gives each step's share.  `dense`: also time
    the dense causal attention of every token (the same attention kernel with
    every KV head keeping all S tokens), the attention the method replaces."""
    from query_adaptive_chunk_b200 import csa
    inp = synth.make_prefill_inputs(w, device="cuda")
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    B, S, Hq, Hkv, D = w.B, w.S, w.Hq, w.Hkv, w.D
    dev = "cuda"
    scale = 1.0 / math.sqrt(D)
    nb = csa.csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    O = torch.empty_like(Q)
    budget = torch.zeros(B, dtype=torch.int32, device=dev)
    # buffers of the separate calls
    U = B * Hkv
    ni = csa.csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs)
    si = torch.empty(ni, dtype=torch.uint8, device=dev)
    imp = torch.empty(B, Hkv, S, device=dev)
    k_seq = torch.empty(B, dtype=torch.int32, device=dev)
    k_unit = torch.empty(U, dtype=torch.int32, device=dev)
    idx = torch.empty(U, S, dtype=torch.int32, device=dev)
    cnt = torch.empty(U, dtype=torch.int32, device=dev)
    Qc, Oc = torch.empty_like(Q), torch.empty_like(Q)
    Kc, Vc = torch.empty_like(K), torch.empty_like(V)
    nd = csa.csa_token_decompress_scratch_bytes(B, S, Hkv)
    sd = torch.empty(nd, dtype=torch.uint8, device=dev)
    O2 = torch.empty_like(Q)
    ev = [_ext_event() for _ in range(len(TOKEN_STAGES) + 1)]

    def whole():
        csa.csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, ws, nb, O,
                                     budget)

    def staged():
        ev[0].record()
        csa.csa_token_importance(Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp, si, ni)
        ev[1].record()
        csa.csa_token_budget(imp, B, S, Hkv, tau, 64, k_seq, k_unit)
        ev[2].record()
        csa.csa_token_select(imp, B, S, Hkv, k_unit, idx, cnt)
        ev[3].record()
        csa.csa_token_compress(Q, K, V, idx, cnt, B, S, Hq, Hkv, D, Qc, Kc, Vc)
        ev[4].record()
        csa.csa_token_attend(Qc, Kc, Vc, k_unit, B, S, Hq, Hkv, D, scale, Oc)
        ev[5].record()
        csa.csa_token_decompress(Oc, idx, cnt, B, S, Hq, Hkv, D, sd, nd, O2)
        ev[6].record()

    for _ in range(warmup):
        whole()
        staged()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=side):
        whole()
    with torch.cuda.graph(g2, stream=side, capture_error_mode="relaxed"):
        staged()
    for _ in range(warmup):
        g1.replay()
        g2.replay()
    torch.cuda.synchronize()
    ms, stage_ms = [], {k: [] for k in TOKEN_STAGES}
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g1.replay()
        e1.record()
        flush()
        g2.replay()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
        for i, k in enumerate(TOKEN_STAGES):
            stage_ms[k].append(ev[i].elapsed_time(ev[i + 1]))
    csa.csa_check_device_status()
    assert torch.equal(O, O2), "the separate calls must give the whole call's output"
    del g1, g2
    dense_ms = []
    if dense:
        k_all = torch.full((U,), S, dtype=torch.int32, device=dev)
        for _ in range(max(1, warmup)):
            csa.csa_token_attend(Q, K, V, k_all, B, S, Hq, Hkv, D, scale, Oc)
        torch.cuda.synchronize()
        for _ in range(max(3, steps // 2)):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            csa.csa_token_attend(Q, K, V, k_all, B, S, Hq, Hkv, D, scale, Oc)
            e1.record()
            torch.cuda.synchronize()
            dense_ms.append(e0.elapsed_time(e1))
        csa.csa_check_device_status()
    k = int(budget.max())
    kt = min(S, (k + 63) // 64 * 64)
    n_t = kt // 64
    # dense causal attention of the kept tokens: tile t sees tiles 0..t
    flops = B * Hkv * (n_t * (n_t + 1) // 2) * w.G * 2 * (2 * 64 * 64 * D)
    n_all = S // 64
    dense_flops = B * Hkv * (n_all * (n_all + 1) // 2) * w.G * 2 * (2 * 64 * 64 * D)
    return {"ms": ms, "stage_ms": stage_ms, "budget": k, "kept_tokens": kt, "flops": flops,
            "n_obs": n_obs, "tau": tau, "dense_ms": dense_ms, "dense_flops": dense_flops}


def token_sparse_line(w, r) -> dict:
    """Bench entry of a Token Sparse run: per-call time, the kept fraction,
    the attention TFLOP/s, and the time of each step with the share of the
    steps other than the dense attention (importance, budget, token choice,
    compress, decompress) in the sum of the steps."""
    ms = statistics.mean(r["ms"])
    st = {k: statistics.mean(v) for k, v in r["stage_ms"].items()}
    tot = sum(st.values())
    return {"ms_per_step": round(ms, 4), "n_obs": r["n_obs"], "tau": r["tau"],
            "budget_tokens": r["budget"], "kept_tokens_per_head": r["kept_tokens"],
            "kept_fraction": round(r["kept_tokens"] / w.S, 4),
            "attention_flops": r["flops"],
            "effective_tflops_whole_step": round(r["flops"] / (ms * 1e-3) / 1e12, 1),
            "attend_tflops": round(r["flops"] / (st["attend"] * 1e-3) / 1e12, 1),
            "stage_ms": {k: round(v, 4) for k, v in st.items()},
            "overhead_share": round((tot - st["attend"]) / tot, 4),
            "importance_budget_share": round((st["importance"] + st["budget"]) / tot, 4),
            **({"dense_attention_ms": round(statistics.mean(r["dense_ms"]), 3),
                "dense_attention_tflops": round(
                    r["dense_flops"] / (statistics.mean(r["dense_ms"]) * 1e-3) / 1e12, 1),
                "speedup_vs_dense_attention": round(statistics.mean(r["dense_ms"]) / ms, 2)}
               if r["dense_ms"] else {})}


def time_token_importance(w, steps: int, warmup: int, flush, n_obs: int = 64, tau: float = 0.1):
    """The first two stages of the Token Sparse call alone on the 32K prefill
    inputs: the proxy importance (csa_token_importance) and the coverage
    budget (csa_token_budget), each between its own events."""
    from query_adaptive_chunk_b200 import csa
    inp = synth.make_prefill_inputs(w, device="cuda")
    Q, K = inp["Q"], inp["K"]
    scale = 1.0 / math.sqrt(w.D)
    imp = torch.empty(w.B, w.Hkv, w.S, dtype=torch.float32, device="cuda")
    nb = csa.csa_token_importance_scratch_bytes(w.B, w.S, w.Hq, w.Hkv, n_obs)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    k_seq = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    k_unit = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")

    def call(e=None):
        if e:
            e[0].record()
        csa.csa_token_importance(Q, K, w.B, w.S, w.Hq, w.Hkv, w.D, n_obs, scale, imp, scratch, nb)
        if e:
            e[1].record()
        csa.csa_token_budget(imp, w.B, w.S, w.Hkv, tau, 64, k_seq, k_unit)
        if e:
            e[2].record()

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    imp_ms, bud_ms = [], []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        call(e)
        torch.cuda.synchronize()
        imp_ms.append(e[0].elapsed_time(e[1]))
        bud_ms.append(e[1].elapsed_time(e[2]))
    csa.csa_check_device_status()
    return {"importance_ms": imp_ms, "budget_ms": bud_ms, "budget": int(k_seq.max())}


def oracle_decode_seconds(w, inp, max_seconds: float = 20.0, max_steps: int = 5, threads: int = 1):
    """The CPU oracle's per-step work (score + select + attention, summaries
    precomputed) on this workload, a bounded number of steps.  threads == 1:
    single-threaded; threads > 1: the units of a step spread over that many
    host threads (numpy releases the GIL inside its array kernels), each
    single-threaded inside."""
    import concurrent.futures as cf

    from threadpoolctl import threadpool_limits

    from oracle import csa_oracle as O
    from oracle import pipeline as OP
    q, K, V = inp["q"].cpu(), inp["K"].cpu(), inp["V"].cpu()
    proj = inp.get("proj")
    projn = None if proj is None else OP.to_np(proj)
    units = synth.decode_units(w)

    def unit_work(bh):
        b, h = bh
        qg = OP.to_np(q[b, h * w.G:(h + 1) * w.G])
        if h in w.full_heads:
            chunks = list(range(w.C))
        else:
            s = O.score_chunks(qg[None, None], summ[(b, h)][None, None], 1, projn)[0, 0, 0]
            if w.select == "topp":
                chunks, _, _ = O.select_topp(s, 1.0 / math.sqrt(w.D), w.p, w.budget,
                                             w.n_sink, w.n_local)
            else:
                chunks, _ = O.select_topk(s, w.k_free, w.n_sink, w.n_local)
        tok = O.chunk_tokens(chunks, w.L)
        ti = torch.as_tensor(tok)
        O.attend(qg, OP.to_np(K[b, h][ti]), OP.to_np(V[b, h][ti]),
                 torch.arange(len(tok)).numpy(), w.scale)

    with threadpool_limits(1):
        summ = {u: OP.unit_summaries(K[u[0], u[1]], w.L, projn) for u in units
                if u[1] not in w.full_heads}
        times = []
        ex = cf.ThreadPoolExecutor(max_workers=threads) if threads > 1 else None
        try:
            t_start = time.perf_counter()
            while len(times) < max_steps and (time.perf_counter() - t_start) < max_seconds:
                t0 = time.perf_counter()
                if ex is None:
                    for u in units:
                        unit_work(u)
                else:
                    list(ex.map(unit_work, units))
                times.append(time.perf_counter() - t0)
        finally:
            if ex is not None:
                ex.shutdown()
    return times


# ---------------------------------------------------------------- arms

def run_reference(args):
    """The CPU oracle timed as the reference arm, on the headline workload."""
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    w = HEADLINE
    inp = synth.make_decode_inputs(w, device="cpu")
    t = oracle_decode_seconds(w, inp, max_seconds=1e9, max_steps=args.warmup + args.steps)
    t = t[args.warmup:] if len(t) > args.warmup else t
    us = 1e6 * statistics.mean(t)
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": "us/step",
            "n_gpus": args.gpus, "steps": len(t), "warmup": args.warmup,
            "ms_per_step": us / 1000, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                       "ctx": w.T, "L": w.L, "select": "top-p p=0.9 cap 256 + sink + 2 local",
                       "full_heads": list(w.full_heads), "proj_rank": w.proj_rank,
                       "timing": "wall clock around each whole oracle step (host)",
                       "parallelism": "one process on the host cores"},
            "cpu_baseline": {"value": us, "unit": "us/step", "cores": 1, "kind": "oracle",
                             "sample": f"{len(t)} whole decode steps of {w.name} (all 8 units), "
                                       "summaries precomputed, numpy fp64 single-threaded",
                             "cpu_model": host_cpu_model(), "host_cores": os.cpu_count()},
            "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_ours(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = dist_init(world, "nccl")
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    flush = make_flush(dev)
    if args.only:
        return run_only(args, flush, load_peaks())

    w = rank_workload(HEADLINE, rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if "CUDA_VISIBLE_DEVICES" in os.environ else local
    with ClockSampler(gpu_index) as clk:
        r = time_decode(w, args.steps, args.warmup, flush)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = clk.summary()
    step_us_local = 1000 * statistics.mean(r["step_ms"])
    step_us = dist_max(step_us_local, world, dev)
    dec_us = 1000 * statistics.mean(r["decode_ms"])
    kv, summ = r["kv_bytes"], r["summ_bytes"]
    step_gbs = (kv + summ) / (step_us * 1e-6) / 1e9
    agg_gbs = dist_sum((kv + summ) / (step_us_local * 1e-6) / 1e9, world, dev)
    dec_gbs = kv / (dec_us * 1e-6) / 1e9
    e2e_graph, e2e_eager, h2d, d2h = time_e2e(w, r["dec"], r["inp"], max(5, args.steps // 2),
                                              flush)
    e2e_eager_us = dist_max(1000 * statistics.mean(e2e_eager), world, dev)
    e2e_us = e2e_eager_us
    e2e_mode = "direct launches per call (query copy, step, output copy)"
    if e2e_graph is not None:
        e2e_us = dist_max(1000 * statistics.mean(e2e_graph), world, dev)
        e2e_mode = "CUDA-graph replay of csa_decode_step_host (query copy, step, output copy)"
    rot = None
    if rank == 0:
        rr = time_decode_rotating(w, r["inp"], max(16, args.steps), args.warmup)
        if rr is not None:
            rot_us = 1000 * statistics.mean(rr["decode_ms"])
            rot = {"decode_us": round(rot_us, 3),
                   "gbs": round(kv / (rot_us * 1e-6) / 1e9, 1),
                   "frac_of_measured_hbm": round(kv / (rot_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                   "step_us": round(1000 * statistics.mean(rr["step_ms"]), 3),
                   "copies": 8, "resident_bytes": 8 * rr["cache_bytes"],
                   "note": "no flush: eight copies of the K/V cache in rotation, each read "
                           "after seven other steps' reads (235.8 MB each) have passed "
                           "through L2; the roofline above keeps the flushed figure"}
    extra = {}
    if rank == 0 and not args.headline_only:
        extra = other_workloads(args, flush, peaks)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t = oracle_decode_seconds(w, r["inp"], max_seconds=20.0, max_steps=5)
        cpu = {"value": 1e6 * statistics.mean(t), "unit": "us/step", "cores": 1, "kind": "oracle",
               "sample": f"{len(t)} whole decode steps of {w.name} (all {w.B * w.Hkv} units), "
                         "summaries precomputed, numpy fp64 single-threaded",
               "cpu_model": host_cpu_model(), "host_cores": os.cpu_count()}
        n_thr = min(os.cpu_count() or 1, w.B * w.Hkv)
        if n_thr > 1:
            tp = oracle_decode_seconds(w, r["inp"], max_seconds=10.0, max_steps=5, threads=n_thr)
            cpu["parallel"] = {"value": 1e6 * statistics.mean(tp), "unit": "us/step",
                               "cores": n_thr, "host_cores": os.cpu_count(),
                               "sample": f"{len(tp)} whole steps, units spread over {n_thr} "
                                         "host threads (one unit per thread)"}
    traffic = recorded_traffic(os.path.join(ROOT, "query_adaptive_chunk_b200", "csrc", "decode.cu"),
                               "decode_bf16_kernel<128,128>/" + w.name)
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": round(step_us, 3), "unit": "us/step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_us / 1000, 6),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "ctx": w.T,
                   "L": w.L, "select": "top-p p=0.9 cap 256 + sink + 2 local",
                   "full_heads": list(w.full_heads), "proj_rank": w.proj_rank,
                   "l2": "flushed before every step (256 MB write + 256 MB read)",
                   "timing": "CUDA-graph replay; step from events captured at the start and "
                             "end of the step inside the graph (device time, the host's graph "
                             "launch excluded: step_with_graph_launch_us includes it); decode "
                             "kernel from events inside a second graph of the same step"
                             if r["graph"] else "direct launches, CUDA events",
                   "parallelism": f"replicas x{world} (units shard, no collective)"},
        "hbm_gbs": round(step_gbs, 1), "hbm_frac_of_measured": round(step_gbs / peaks["hbm_gbs"], 4),
        "hbm_frac_of_8tbs_nominal": round(step_gbs / 8000.0, 4),
        "aggregate_hbm_gbs": round(agg_gbs, 1),
        "step_bytes": {"selected_kv": kv, "summaries": summ, "chunks": r["chunks"]},
        "roofline": {"kernel": "decode_bf16_kernel<128,128> (merged split-K decode)", "bound": "hbm",
                     "achieved": round(dec_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(dec_gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "algorithmic_bytes": kv, "duration_us": round(dec_us, 3),
                     "peak_source": peaks["source"]},
        "e2e": {"value": round(e2e_us, 3), "unit": "us/step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "mode": e2e_mode,
                "direct_launch_value": round(e2e_eager_us, 3)},
        "gpu_launches": 2 * args.steps,
        "step_with_graph_launch_us": round(1000 * statistics.mean(r["step_with_launch_ms"]), 3),
        "select_us": round(1000 * statistics.mean(r["select_ms"]), 3),
        "decode_inputs_larger_than_l2": rot,
        "timing_stats": {"rank": 0, "step_us_median": round(1000 * statistics.median(r["step_ms"]), 3),
                         "step_us_min": round(1000 * min(r["step_ms"]), 3),
                         "decode_us_median": round(1000 * statistics.median(r["decode_ms"]), 3),
                         "decode_us_min": round(1000 * min(r["decode_ms"]), 3)},
        "clocks": clocks,
        "cpu_baseline": cpu,
        "workloads": extra,
    }
    print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def other_workloads(args, flush, peaks):
    out = {}
    steps = max(5, args.steps // 2)
    # the tensor-core prefill first: the 128K Token Sparse line below runs
    # ~0.6 s of dense attention, after which the GPU sits at its power cap
    w = synth.PREFILL_32K
    r = time_prefill(w, steps, args.warmup, flush)
    att_ms = statistics.mean(r["attend_ms"])
    tflops = r["flops"] / (att_ms * 1e-3) / 1e12
    out[w.name] = {"attend_ms": round(att_ms, 4), "select_ms": round(statistics.mean(r["select_ms"]), 4),
                   "executed_blocks": r["blocks"], "flops": r["flops"],
                   "tflops": round(tflops, 1),
                   "frac_of_measured_bf16": round(tflops / peaks["bf16_tflops"], 4),
                   "frac_of_sustained_bf16": round(tflops / peaks["bf16_tflops_sustained"], 4),
                   "frac_of_2250_nominal_bf16": round(tflops / 2250.0, 4),
                   "diagonal_blocks": r["diagonal_blocks"],
                   "causal_effective_flops": int(r["causal_flops"]),
                   "causal_effective_tflops": round(r["causal_flops"] / (att_ms * 1e-3) / 1e12, 1)}
    del r
    torch.cuda.empty_cache()
    for w in (synth.TOPK_32K, synth.HIER_1M, synth.TINY_F32, synth.TOPK_UNION_32K,
              synth.HYBRID_TOPK_32K, synth.HYBRID_ALL_TOPK_32K, synth.ROPE_TOPK_32K):
        r = time_decode(w, steps, args.warmup, flush)
        us = 1000 * statistics.mean(r["step_ms"])
        dus = 1000 * statistics.mean(r["decode_ms"])
        byt = r["kv_bytes"] + r["summ_bytes"]
        out[w.name] = {"us_per_step": round(us, 3), "step_gbs": round(byt / (us * 1e-6) / 1e9, 1),
                       "us_per_step_with_graph_launch": round(
                           1000 * statistics.mean(r["step_with_launch_ms"]), 3),
                       "step_frac_of_measured_hbm": round(byt / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                       "decode_us": round(dus, 3),
                       "decode_gbs": round(r["kv_bytes"] / (dus * 1e-6) / 1e9, 1),
                       "decode_frac_of_measured_hbm": round(
                           r["kv_bytes"] / (dus * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                       "select_us": round(1000 * statistics.mean(r["select_ms"]), 3),
                       "selected_kv_bytes": r["kv_bytes"], "summary_bytes": r["summ_bytes"]}
        if w in (synth.TOPK_32K, synth.HIER_1M):
            # the same steps with inputs larger than L2 instead of the flush
            # 16 copies of the 1M cache: 15 other steps' 18 MB pass between two reads
            n_cp = 16 if w is synth.HIER_1M else 8
            rr = time_decode_rotating(w, r["inp"], max(2 * n_cp, steps), args.warmup, n_cp)
            if rr is not None:
                su, du = 1000 * statistics.mean(rr["step_ms"]), 1000 * statistics.mean(rr["decode_ms"])
                out[w.name]["inputs_larger_than_l2"] = {
                    "us_per_step": round(su, 3), "decode_us": round(du, 3),
                    "decode_frac_of_measured_hbm": round(
                        r["kv_bytes"] / (du * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                    "copies": n_cp, "resident_bytes": n_cp * rr["cache_bytes"],
                    "note": f"no flush: {n_cp} copies of the K/V cache in rotation"}
            del rr
        del r
        torch.cuda.empty_cache()
    # the headline step as the separate boundary calls (split partials and the
    # stand-alone log-sum-exp merge)
    r = time_separate_calls(synth.TOPP_128K, steps, args.warmup, flush)
    if r is not None:
        st = {k: 1000 * statistics.mean(v) for k, v in r["ms"].items()}
        kv = selected_bytes(synth.TOPP_128K, r["dec"])[0]
        out["topp_mixed_decode_bf16_ctx128k_separate_calls"] = {
            "score_us": round(st["score"], 3), "select_us": round(st["select"], 3),
            "decode_split_partials_us": round(st["decode"], 3), "merge_us": round(st["merge"], 3),
            "sum_us": round(st["score"] + st["select"] + st["decode"] + st["merge"], 3),
            "decode_then_merge_us": round(st["decode_merge"], 3),
            "decode_gbs": round(kv / (st["decode"] * 1e-6) / 1e9, 1),
            "decode_frac_of_measured_hbm": round(kv / (st["decode"] * 1e-6) / 1e9 /
                                                 peaks["hbm_gbs"], 4),
            "merge_read_bytes": r["merge_read_bytes"],
            "merge_gbs": round(r["merge_read_bytes"] / (st["merge"] * 1e-6) / 1e9, 1)}
        del r
        torch.cuda.empty_cache()
    for tw, name in ((synth.PREFILL_32K, "token_sparse_prefill_bf16_seq32k"),
                     (synth.TOKEN_SPARSE_HEAVY_32K, synth.TOKEN_SPARSE_HEAVY_32K.name),
                     (synth.TOKEN_SPARSE_HEAVY_128K, synth.TOKEN_SPARSE_HEAVY_128K.name)):
        r = time_token_sparse(tw, steps, args.warmup, flush,
                              dense=tw is synth.TOKEN_SPARSE_HEAVY_128K)
        out[name] = token_sparse_line(tw, r)
        del r
        torch.cuda.empty_cache()
    return out


def run_only(args, flush, peaks):
    """Time one named workload alone and print its figures (profiling aid)."""
    if args.only == synth.TOKEN_SPARSE_HEAVY_128K.name:
        tw = synth.TOKEN_SPARSE_HEAVY_128K
        r = time_token_sparse(tw, args.steps, args.warmup, flush, dense=True)
        print(json.dumps({"workload": args.only, **token_sparse_line(tw, r)}))
        return 0
    if args.only in ("token_sparse_prefill_bf16_seq32k", synth.TOKEN_SPARSE_HEAVY_32K.name):
        tw = synth.PREFILL_32K if args.only == "token_sparse_prefill_bf16_seq32k" else \
            synth.TOKEN_SPARSE_HEAVY_32K
        r = time_token_sparse(tw, args.steps, args.warmup, flush)
        print(json.dumps({"workload": args.only, **token_sparse_line(tw, r)}))
        return 0
    if args.only == "token_importance_bf16_seq32k":
        r = time_token_importance(synth.PREFILL_32K, args.steps, args.warmup, flush)
        print(json.dumps({"workload": args.only,
                          "importance_ms": statistics.mean(r["importance_ms"]),
                          "budget_ms": statistics.mean(r["budget_ms"]), "budget": r["budget"]}))
        return 0
    byname = {w.name: w for w in synth.ALL_WORKLOADS}
    w = byname[args.only]
    if isinstance(w, synth.PrefillWorkload):
        r = time_prefill(w, args.steps, args.warmup, flush)
        ms = statistics.mean(r["attend_ms"])
        d = {"workload": w.name, "attend_ms": ms, "tflops": r["flops"] / (ms * 1e-3) / 1e12,
             "select_ms": statistics.mean(r["select_ms"])}
    else:
        r = time_decode(w, args.steps, args.warmup, flush)
        us = 1000 * statistics.mean(r["step_ms"])
        dus = 1000 * statistics.mean(r["decode_ms"])
        d = {"workload": w.name, "us_per_step": us, "decode_us": dus,
             "select_us": 1000 * statistics.mean(r["select_ms"]),
             "decode_gbs": r["kv_bytes"] / (dus * 1e-6) / 1e9}
    print(json.dumps(d))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None, help="time one named workload alone")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
