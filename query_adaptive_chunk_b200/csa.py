"""Python binding of libcsa.so (the C ABI in include/csa.h).

Argument marshalling only: each function has the name and the positional
arguments of its C counterpart, accepts torch tensors (their data pointers
are passed), ``None`` for NULL, and an optional ``stream`` (default: torch's
current CUDA stream).  A non-OK status raises ``CsaError`` with the library's
message.  Every step of the method runs in the library's CUDA kernels; there
is no fallback when the library is missing: importing this module fails.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "csa.h")

CSA_F32, CSA_BF16 = 0, 1
STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CUDA",
          4: "CSA_ERR_TIMEOUT", 5: "CSA_ERR_DEVICE_INDEX"}


class CsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {message}")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m query_adaptive_chunk_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _i64, _f, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64
_SIGS = {
    "csa_version": (_i, []),
    "csa_last_error_string": (ctypes.c_char_p, []),
    "csa_check_device_status": (_i, [_vp]),
    "csa_set_wait_limit_ns": (None, [_u64]),
    "csa_get_wait_limit_ns": (_u64, []),
    "csa_selftest_wait_timeout": (_i, [_u64, _vp]),
    "csa_chunk_summaries": (_i, [_vp, _i, _i, _i, _i64, _i, _i, _vp, _i, _vp, _vp]),
    "csa_meta_summaries": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "csa_tile_mean_q": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp]),
    "csa_rope": (_i, [_vp, _vp, _i, _i64, _i, _i64, _i64, _f, _vp]),
    "csa_token_importance_scratch_bytes": (_i64, [_i, _i, _i, _i, _i]),
    "csa_token_importance": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp, _i64, _vp]),
    "csa_token_budget": (_i, [_vp, _i, _i, _i, _f, _i, _vp, _vp, _vp]),
    "csa_token_sparse_workspace_bytes": (_i64, [_i, _i, _i, _i, _i, _i]),
    "csa_token_sparse_prefill": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _f, _vp, _i64,
                                      _vp, _vp, _vp]),
    "csa_token_select": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "csa_token_compress": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "csa_token_attend": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp]),
    "csa_token_decompress_scratch_bytes": (_i64, [_i, _i, _i]),
    "csa_token_decompress": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i64, _vp, _vp]),
    "csa_score_chunks": (_i, [_vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _i, _vp,
                              _vp]),
    "csa_select_topk": (_i, [_vp, _i, _i, _vp, _i, _i, _i, _vp, _vp, _i, _vp]),
    "csa_select_topk_causal": (_i, [_vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _i, _vp]),
    "csa_select_topp": (_i, [_vp, _i, _i, _f, _f, _i, _i, _i, _vp, _vp, _i, _vp, _vp]),
    "csa_select_hier": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp,
                             _i, _vp]),
    "csa_sparse_decode": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i64, _i, _f,
                               _i, _i, _vp, _vp, _vp]),
    "csa_decode_default_parts": (_i, [_i, _i, _i]),
    "csa_score_select_topk": (_i, [_vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _i, _i, _i,
                                   _vp, _vp, _i, _vp]),
    "csa_score_select_topk_union": (_i, [_vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _i, _i,
                                         _i, _vp, _vp, _i, _vp]),
    "csa_score_select_topp": (_i, [_vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _f, _f, _i,
                                   _i, _i, _vp, _vp, _i, _vp, _vp]),
    "csa_decode_workspace_bytes": (_i64, [_i, _i, _i, _i, _i]),
    "csa_sparse_decode_merged": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i64,
                                      _i, _f, _i, _vp, _i64, _vp, _i, _vp, _vp]),
    "csa_sparse_decode_merged_hybrid": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _vp, _i, _vp,
                                             _i, _i, _i, _i, _i64, _i, _f, _i, _vp, _i64, _vp,
                                             _i, _vp, _vp]),
    "csa_sparse_decode_merged_noalloc": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _i, _vp, _i, _i, _i, _i,
                                              _i64, _i, _f, _i, _vp, _i, _vp, _vp]),
    "csa_lse_merge": (_i, [_vp, _vp, _i, _i, _i, _vp, _i, _vp, _vp]),
    "csa_decode_step": (_i, [_vp, _vp]),
    "csa_decode_step_host": (_i, [_vp, _vp, _vp, _vp, _vp]),
    "csa_block_sparse_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                      _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_functions() -> list:
    """Names of the functions include/csa.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"CSA_API\s+[\w\s\*]*?\b(csa_\w+)\s*\(", text)))


def _p(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return ctypes.c_void_p(x.data_ptr())
    return ctypes.c_void_p(int(x))


def _s(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dt(d) -> int:
    if isinstance(d, torch.dtype):
        return {torch.float32: CSA_F32, torch.bfloat16: CSA_BF16}[d]
    return int(d)


def _check(status: int):
    if status != 0:
        raise CsaError(status, lib.csa_last_error_string().decode())


def csa_version() -> int:
    return lib.csa_version()


def csa_last_error_string() -> str:
    return lib.csa_last_error_string().decode()


def csa_check_device_status(stream=None) -> None:
    _check(lib.csa_check_device_status(_s(stream)))


def csa_set_wait_limit_ns(ns: int) -> None:
    lib.csa_set_wait_limit_ns(int(ns))


def csa_get_wait_limit_ns() -> int:
    return lib.csa_get_wait_limit_ns()


def csa_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib.csa_selftest_wait_timeout(int(limit_ns), _s(stream)))


def csa_chunk_summaries(K, dtype, B, Hkv, T, D, L, proj, R, summ, stream=None):
    _check(lib.csa_chunk_summaries(_p(K), _dt(dtype), B, Hkv, T, D, L, _p(proj), R, _p(summ),
                                   _s(stream)))


def csa_meta_summaries(summ, B, Hkv, C, Ds, Gm, meta, stream=None):
    _check(lib.csa_meta_summaries(_p(summ), B, Hkv, C, Ds, Gm, _p(meta), _s(stream)))


def csa_tile_mean_q(Q, dtype, B, S, Hq, D, tile_m, qbar, stream=None):
    _check(lib.csa_tile_mean_q(_p(Q), _dt(dtype), B, S, Hq, D, tile_m, _p(qbar), _s(stream)))


def csa_score_chunks(q, q_dtype, proj, R, summ, B, Nq, Hq, Hkv, D, C, head_full, causal_tile_m,
                     causal_L, scores, stream=None):
    _check(lib.csa_score_chunks(_p(q), _dt(q_dtype), _p(proj), R, _p(summ), B, Nq, Hq, Hkv, D, C,
                                _p(head_full), causal_tile_m, causal_L, _p(scores), _s(stream)))


def csa_select_topk(scores, U, C, n_valid, k_free, n_sink, n_local, idx, count, kmax, stream=None):
    _check(lib.csa_select_topk(_p(scores), U, C, _p(n_valid), k_free, n_sink, n_local, _p(idx),
                               _p(count), kmax, _s(stream)))


def csa_select_topk_causal(scores, U, C, n_tiles, tile_m, L, k_free, n_sink, n_local, idx, count,
                           kmax, stream=None):
    _check(lib.csa_select_topk_causal(_p(scores), U, C, n_tiles, tile_m, L, k_free, n_sink,
                                      n_local, _p(idx), _p(count), kmax, _s(stream)))


def csa_select_topp(scores, U, C, logit_scale, p, budget, n_sink, n_local, idx, count, kmax,
                    n_p_out=None, stream=None):
    _check(lib.csa_select_topp(_p(scores), U, C, logit_scale, p, budget, n_sink, n_local, _p(idx),
                               _p(count), kmax, _p(n_p_out), _s(stream)))


def csa_select_hier(q, q_dtype, meta, summ, B, Hq, Hkv, D, C, Gm, top_meta, k_free, n_sink,
                    n_local, idx, count, kmax, stream=None):
    _check(lib.csa_select_hier(_p(q), _dt(q_dtype), _p(meta), _p(summ), B, Hq, Hkv, D, C, Gm,
                               top_meta, k_free, n_sink, n_local, _p(idx), _p(count), kmax,
                               _s(stream)))


def csa_sparse_decode(q, K, V, dtype, idx, count, kmax, head_full, B, Hq, Hkv, D, T, L, scale,
                      num_parts, max_splits, o_part, lse_part, stream=None):
    _check(lib.csa_sparse_decode(_p(q), _p(K), _p(V), _dt(dtype), _p(idx), _p(count), kmax,
                                 _p(head_full), B, Hq, Hkv, D, T, L, scale, num_parts, max_splits,
                                 _p(o_part), _p(lse_part), _s(stream)))


def csa_decode_default_parts(dtype, D, L) -> int:
    n = lib.csa_decode_default_parts(_dt(dtype), D, L)
    if n < 0:
        raise CsaError(3, csa_last_error_string())
    return n


def csa_score_select_topk(q, q_dtype, proj, R, summ, B, Hq, Hkv, D, C, head_full, k_free, n_sink,
                          n_local, idx, count, kmax, stream=None):
    _check(lib.csa_score_select_topk(_p(q), _dt(q_dtype), _p(proj), R, _p(summ), B, Hq, Hkv, D, C,
                                     _p(head_full), k_free, n_sink, n_local, _p(idx), _p(count),
                                     kmax, _s(stream)))


def csa_score_select_topk_union(q, q_dtype, proj, R, summ, B, Hq, Hkv, D, C, head_full, k_free,
                                n_sink, n_local, idx, count, kmax, stream=None):
    _check(lib.csa_score_select_topk_union(_p(q), _dt(q_dtype), _p(proj), R, _p(summ), B, Hq, Hkv,
                                           D, C, _p(head_full), k_free, n_sink, n_local, _p(idx),
                                           _p(count), kmax, _s(stream)))


def csa_score_select_topp(q, q_dtype, proj, R, summ, B, Hq, Hkv, D, C, head_full, logit_scale, p,
                          budget, n_sink, n_local, idx, count, kmax, n_p_out=None, stream=None):
    _check(lib.csa_score_select_topp(_p(q), _dt(q_dtype), _p(proj), R, _p(summ), B, Hq, Hkv, D, C,
                                     _p(head_full), logit_scale, p, budget, n_sink, n_local,
                                     _p(idx), _p(count), kmax, _p(n_p_out), _s(stream)))


def csa_rope(x, y, dtype, rows, D, period, pos0, theta, stream=None):
    """Rotary position embedding of x [rows, D] into y (may be x): row r at
    position pos0 + r % period (see include/csa.h)."""
    _check(lib.csa_rope(_p(x), _p(y), _dt(dtype), rows, D, period, pos0, theta, _s(stream)))


def csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs) -> int:
    n = lib.csa_token_importance_scratch_bytes(B, S, Hq, Hkv, n_obs)
    if n < 0:
        raise CsaError(1, "csa_token_importance_scratch_bytes: bad sizes")
    return n


def csa_token_importance(Q, K, B, S, Hq, Hkv, D, n_obs, scale, imp, scratch, scratch_bytes,
                         stream=None):
    _check(lib.csa_token_importance(_p(Q), _p(K), B, S, Hq, Hkv, D, n_obs, scale, _p(imp),
                                    _p(scratch), scratch_bytes, _s(stream)))


def csa_token_budget(imp, B, S, Hkv, tau, tile, k_seq, k_unit, stream=None):
    _check(lib.csa_token_budget(_p(imp), B, S, Hkv, tau, tile, _p(k_seq), _p(k_unit), _s(stream)))


def csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs) -> int:
    n = lib.csa_token_sparse_workspace_bytes(B, S, Hq, Hkv, D, n_obs)
    if n < 0:
        raise CsaError(1, "csa_token_sparse_workspace_bytes: bad sizes")
    return n


def csa_token_sparse_prefill(Q, K, V, B, S, Hq, Hkv, D, n_obs, tau, scale, workspace,
                             workspace_bytes, O, budget_out, stream=None):
    """Token Sparse Attention prefill: importance, coverage budget, each KV
    head's own tokens, dense causal attention of the compressed sequences,
    scatter back (see include/csa.h)."""
    _check(lib.csa_token_sparse_prefill(_p(Q), _p(K), _p(V), B, S, Hq, Hkv, D, n_obs, tau, scale,
                                        _p(workspace), workspace_bytes, _p(O), _p(budget_out),
                                        _s(stream)))


def csa_token_select(imp, B, S, Hkv, k_unit, idx, count, stream=None):
    _check(lib.csa_token_select(_p(imp), B, S, Hkv, _p(k_unit), _p(idx), _p(count), _s(stream)))


def csa_token_compress(Q, K, V, idx, count, B, S, Hq, Hkv, D, Qc, Kc, Vc, stream=None):
    _check(lib.csa_token_compress(_p(Q), _p(K), _p(V), _p(idx), _p(count), B, S, Hq, Hkv, D,
                                  _p(Qc), _p(Kc), _p(Vc), _s(stream)))


def csa_token_attend(Qc, Kc, Vc, k_unit, B, S, Hq, Hkv, D, scale, Oc, stream=None):
    _check(lib.csa_token_attend(_p(Qc), _p(Kc), _p(Vc), _p(k_unit), B, S, Hq, Hkv, D, scale,
                                _p(Oc), _s(stream)))


def csa_token_decompress_scratch_bytes(B, S, Hkv) -> int:
    return int(lib.csa_token_decompress_scratch_bytes(B, S, Hkv))


def csa_token_decompress(Oc, idx, count, B, S, Hq, Hkv, D, scratch, scratch_bytes, O,
                         stream=None):
    _check(lib.csa_token_decompress(_p(Oc), _p(idx), _p(count), B, S, Hq, Hkv, D, _p(scratch),
                                    scratch_bytes, _p(O), _s(stream)))


def csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts) -> int:
    n = lib.csa_decode_workspace_bytes(B, Hq, Hkv, D, num_parts)
    if n < 0:
        raise CsaError(1, "csa_decode_workspace_bytes: bad sizes")
    return n


def csa_sparse_decode_merged(q, K, V, dtype, idx, count, kmax, head_full, B, Hq, Hkv, D, T, L,
                             scale, num_parts, workspace, workspace_bytes, out, out_dtype, lse_out,
                             stream=None):
    _check(lib.csa_sparse_decode_merged(_p(q), _p(K), _p(V), _dt(dtype), _p(idx), _p(count), kmax,
                                        _p(head_full), B, Hq, Hkv, D, T, L, scale, num_parts,
                                        _p(workspace), workspace_bytes, _p(out), _dt(out_dtype),
                                        _p(lse_out), _s(stream)))


CSA_GIST_SELECTED, CSA_GIST_ALL = 0, 1


def _scope(gist_scope) -> int:
    if isinstance(gist_scope, str):
        return {"selected": CSA_GIST_SELECTED, "all": CSA_GIST_ALL}[gist_scope]
    return int(gist_scope)


def csa_sparse_decode_merged_hybrid(q, K, V, Kg, Vg, gist_scope, dtype, idx, count, kmax,
                                    head_full, B, Hq, Hkv, D, T, L, scale, num_parts, workspace,
                                    workspace_bytes, out, out_dtype, lse_out, stream=None):
    """The merged decode over the hybrid context: the raw KV of the selected
    chunks plus gist K/V rows (Kg, Vg [B, Hkv, T/L, D]) of the selected chunks
    (gist_scope "selected" / CSA_GIST_SELECTED) or of every chunk ("all" /
    CSA_GIST_ALL); see include/csa.h."""
    _check(lib.csa_sparse_decode_merged_hybrid(_p(q), _p(K), _p(V), _p(Kg), _p(Vg),
                                               _scope(gist_scope), _dt(dtype),
                                               _p(idx), _p(count), kmax, _p(head_full), B, Hq,
                                               Hkv, D, T, L, scale, num_parts, _p(workspace),
                                               workspace_bytes, _p(out), _dt(out_dtype),
                                               _p(lse_out), _s(stream)))


def csa_sparse_decode_merged_noalloc(q, K, V, dtype, idx, count, kmax, head_full, B, Hq, Hkv, D,
                                     T, L, scale, num_parts, out, out_dtype, lse_out, stream=None):
    """csa_sparse_decode_merged without a workspace: the library's built-in
    16 MiB scratch is used, so nothing is allocated (see include/csa.h)."""
    _check(lib.csa_sparse_decode_merged_noalloc(_p(q), _p(K), _p(V), _dt(dtype), _p(idx),
                                                _p(count), kmax, _p(head_full), B, Hq, Hkv, D, T,
                                                L, scale, num_parts, _p(out), _dt(out_dtype),
                                                _p(lse_out), _s(stream)))


CSA_SELECT_TOPK, CSA_SELECT_TOPP, CSA_SELECT_HIER, CSA_SELECT_TOPK_UNION = 0, 1, 2, 3


class DecodeStepDesc(ctypes.Structure):
    """ctypes mirror of csa_decode_step_desc (field order and types as in
    include/csa.h)."""
    _fields_ = [
        ("q", _vp), ("K", _vp), ("V", _vp),
        ("B", _i), ("Hq", _i), ("Hkv", _i), ("D", _i),
        ("T", _i64), ("L", _i), ("scale", _f), ("head_full", _vp),
        ("mode", _i), ("summ", _vp), ("proj", _vp), ("R", _i), ("meta", _vp),
        ("Gm", _i), ("top_meta", _i), ("k_free", _i), ("n_sink", _i), ("n_local", _i),
        ("logit_scale", _f), ("p", _f), ("budget", _i),
        ("idx", _vp), ("count", _vp), ("kmax", _i), ("n_p_out", _vp),
        ("num_parts", _i), ("workspace", _vp), ("workspace_bytes", _i64),
        ("out", _vp), ("out_dtype", _i), ("lse_out", _vp),
        ("Kg", _vp), ("Vg", _vp), ("gist_scope", _i), ("q_score", _vp),
    ]


def decode_step_desc(**kw) -> DecodeStepDesc:
    """Build a descriptor; tensors become their data pointers, dtypes their codes."""
    d = DecodeStepDesc()
    for k, v in kw.items():
        if k == "out_dtype":
            v = _dt(v)
        elif k == "gist_scope":
            v = _scope(v)
        elif isinstance(v, torch.Tensor) or (v is None and k not in ("scale", "p")):
            v = None if v is None else v.data_ptr()
        setattr(d, k, v)
    return d


def csa_decode_step(desc: DecodeStepDesc, stream=None):
    _check(lib.csa_decode_step(ctypes.byref(desc), _s(stream)))


def csa_decode_step_host(desc: DecodeStepDesc, q_host, out_host, lse_host=None, stream=None):
    _check(lib.csa_decode_step_host(ctypes.byref(desc), _p(q_host), _p(out_host), _p(lse_host),
                                    _s(stream)))


def csa_lse_merge(o_part, lse_part, rows, max_splits, D, out, out_dtype, lse_out, stream=None):
    _check(lib.csa_lse_merge(_p(o_part), _p(lse_part), rows, max_splits, D, _p(out),
                             _dt(out_dtype), _p(lse_out), _s(stream)))


def csa_block_sparse_prefill(Q, K, V, idx, count, kmax, B, S, Hq, Hkv, D, tile_m, L, scale, O,
                             stream=None):
    _check(lib.csa_block_sparse_prefill(_p(Q), _p(K), _p(V), _p(idx), _p(count), kmax, B, S, Hq,
                                        Hkv, D, tile_m, L, scale, _p(O), _s(stream)))
