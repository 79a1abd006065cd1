"""The C-ABI library builds, loads, exports every function include/csa.h
declares, and rejects invalid arguments on the host before any CUDA call.
No kernel runs here (these tests need no GPU)."""
import ctypes
import os
import subprocess

import pytest

from query_adaptive_chunk_b200 import build as B


@pytest.fixture(scope="module")
def csa():
    if not os.path.exists(B.LIB) or any(os.path.getmtime(s) > os.path.getmtime(B.LIB)
                                        for s in B.sources()):
        B.build()
    from query_adaptive_chunk_b200 import csa as mod
    return mod


def test_header_declares_the_boundary(csa):
    names = csa.header_functions()
    for n in ["csa_score_chunks", "csa_select_topk", "csa_select_topp", "csa_select_hier",
              "csa_sparse_decode", "csa_lse_merge", "csa_block_sparse_prefill",
              "csa_chunk_summaries", "csa_meta_summaries", "csa_tile_mean_q"]:
        assert n in names


def test_every_declared_symbol_is_exported(csa):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for n in csa.header_functions():
        assert n in exported, n
        assert hasattr(csa.lib, n)
    assert csa.csa_version() == 10000


def test_invalid_arguments_rejected_on_host(csa):
    lib = csa.lib
    null = None
    s0 = ctypes.c_void_p(0)
    # kmax must be positive
    assert lib.csa_select_topk(null, 1, 10, null, 2, 1, 1, null, null, 0, s0) == 1
    assert "kmax" in csa.csa_last_error_string()
    # kmax smaller than the largest possible set
    assert lib.csa_select_topk(null, 1, 10, null, 4, 1, 1, null, null, 5, s0) == 1
    # p outside (0, 1]
    assert lib.csa_select_topp(null, 1, 10, 1.0, 1.5, 4, 1, 1, null, null, 8, null, s0) == 1
    # head dim the decode kernels do not implement
    assert lib.csa_sparse_decode(null, null, null, 1, null, null, 4, null, 1, 4, 1, 96, 1024, 64,
                                 0.1, 0, 148, null, null, s0) == 2
    # chunk length that does not divide the context
    assert lib.csa_sparse_decode(null, null, null, 1, null, null, 4, null, 1, 4, 1, 128, 1000, 64,
                                 0.1, 0, 148, null, null, s0) == 1
    # GQA group size > 8
    assert lib.csa_sparse_decode(null, null, null, 1, null, null, 4, null, 1, 16, 1, 128, 1024, 64,
                                 0.1, 0, 148, null, null, s0) == 2
    # merge width not a multiple of 4
    assert lib.csa_lse_merge(null, null, 4, 8, 6, null, 0, null, s0) == 2
    # prefill shapes outside the implemented tcgen05 tile
    assert lib.csa_block_sparse_prefill(null, null, null, null, null, 18, 1, 4096, 32, 8, 64, 64,
                                        64, 0.1, null, s0) == 2
    # bad dtype code
    assert lib.csa_chunk_summaries(null, 7, 1, 1, 1024, 128, 64, null, 0, null, s0) == 1
    # summary width the score kernel does not implement
    assert lib.csa_score_chunks(null, 1, null, 0, null, 1, 1, 4, 1, 96, 16, null, 0, 0, null,
                                s0) == 2


def test_wait_limit_setting(csa):
    old = csa.csa_get_wait_limit_ns()
    try:
        csa.csa_set_wait_limit_ns(123456)
        assert csa.csa_get_wait_limit_ns() == 123456
    finally:
        csa.csa_set_wait_limit_ns(old)


def test_decode_step_descriptor_layout(csa):
    """The ctypes mirror of csa_decode_step_desc has the C struct's size and
    field offsets (compiled from include/csa.h by the host compiler)."""
    import tempfile
    fields = [f for f, _ in csa.DecodeStepDesc._fields_]
    prog = ['#include <stdio.h>', '#include <stddef.h>', '#include "csa.h"', 'int main(void) {',
            '  printf("%zu\\n", sizeof(csa_decode_step_desc));']
    prog += [f'  printf("%zu\\n", offsetof(csa_decode_step_desc, {f}));' for f in fields]
    prog += ['  return 0;', '}']
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(B.__file__))), "include")
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        with open(src, "w") as f:
            f.write("\n".join(prog) + "\n")
        subprocess.run(["gcc", "-I", inc, src, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                               check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(csa.DecodeStepDesc)
    for f, off in zip(fields, vals[1:]):
        assert getattr(csa.DecodeStepDesc, f).offset == off, f


def test_decode_step_rejects_on_host(csa):
    d = csa.decode_step_desc(B=1, Hq=4, Hkv=1, D=128, T=1024, L=64, scale=0.1, mode=7, kmax=4)
    assert csa.lib.csa_decode_step(ctypes.byref(d), ctypes.c_void_p(0)) == 1
    assert "mode" in csa.csa_last_error_string()
    assert csa.lib.csa_decode_step(None, ctypes.c_void_p(0)) == 1


def test_decode_step_host_rejects_on_host(csa):
    """csa_decode_step_host refuses a missing descriptor and the RoPE-aware
    split (q_score set) before touching any buffer."""
    lib = csa.lib
    s0 = ctypes.c_void_p(0)
    assert lib.csa_decode_step_host(None, None, None, None, s0) == 1
    assert "descriptor" in csa.csa_last_error_string()
    d = csa.decode_step_desc(B=1, Hq=4, Hkv=1, D=128, T=1024, L=64, scale=0.1, mode=0, kmax=4)
    d.q_score = 4096
    assert lib.csa_decode_step_host(ctypes.byref(d), None, None, None, s0) == 2
    assert "q_score" in csa.csa_last_error_string()
    d.q_score = None
    # NULL host buffers
    assert lib.csa_decode_step_host(ctypes.byref(d), None, None, None, s0) == 1
    assert "q_host" in csa.csa_last_error_string()
