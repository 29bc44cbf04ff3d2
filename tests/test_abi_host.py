"""The C ABI without a GPU: the library loads, exports every function that
include/kld.h declares, and rejects bad arguments on the host before any
CUDA call (so these run on a CPU-only machine)."""
import ctypes
import os
import re

import pytest

from quantization_fidelity_scoring_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    with open(os.path.join(ROOT, "include", "kld.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(kld_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from quantization_fidelity_scoring_b200 import build
        build.build()
    return _lib.load()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"kld_full_vocab", "kld_topk_tail", "kld_reduce_stats"} <= set(names)
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.PROTOTYPES, f"binding lacks a prototype for {name}"


def test_status_strings(lib):
    for s in range(6):
        assert lib.kld_status_string(s)
    assert lib.kld_version() >= 100


def test_stats_struct_size_matches_header():
    assert ctypes.sizeof(_lib.KldStats) == 280


A16 = 1 << 20          # a fake, 16-byte aligned "device" address; never dereferenced
MIS = A16 + 4          # 4-byte aligned only


def fv(lib, **kw):
    a = dict(ref=A16, cand=A16 + 4096, dtype=_lib.KLD_BF16, n=4, V=64, ldr=64, ldc=64, tgt=None,
             kl=A16 + 8192, ra=None, ca=None, lpr=None, lpc=None, ws=A16 + 65536, wsb=None, st=None)
    a.update(kw)
    wsb = lib.kld_full_vocab_workspace_size(max(a["n"], 0)) if a["wsb"] is None else a["wsb"]
    return lib.kld_full_vocab(a["ref"], a["cand"], a["dtype"], a["n"], a["V"], a["ldr"], a["ldc"],
                              a["tgt"], a["kl"], a["ra"], a["ca"], a["lpr"], a["lpc"], a["ws"], wsb,
                              a["st"], None)


def test_full_vocab_validation(lib):
    assert fv(lib, dtype=7) == _lib.KLD_ERR_UNSUPPORTED
    assert fv(lib, n=-1) == _lib.KLD_ERR_INVALID_ARG
    assert fv(lib, V=0) == _lib.KLD_ERR_INVALID_ARG
    assert fv(lib, ldr=32) == _lib.KLD_ERR_INVALID_ARG
    assert fv(lib, ref=None) == _lib.KLD_ERR_INVALID_ARG
    assert fv(lib, kl=None) == _lib.KLD_ERR_INVALID_ARG
    assert fv(lib, lpr=A16) == _lib.KLD_ERR_INVALID_ARG          # target lp without target ids
    assert fv(lib, ref=MIS) == _lib.KLD_ERR_ALIGNMENT
    assert fv(lib, ldr=68, V=64) == _lib.KLD_ERR_ALIGNMENT        # 136 B rows
    assert fv(lib, dtype=_lib.KLD_F32, ldr=66) == _lib.KLD_ERR_ALIGNMENT
    assert fv(lib, kl=A16 + 2) == _lib.KLD_ERR_ALIGNMENT
    assert fv(lib, ws=None) == _lib.KLD_ERR_WORKSPACE
    assert fv(lib, wsb=64) == _lib.KLD_ERR_WORKSPACE
    assert fv(lib, ws=A16 + 16) == _lib.KLD_ERR_ALIGNMENT
    assert fv(lib, n=0) == _lib.KLD_OK                            # nothing to launch
    assert fv(lib, n=0, ref=None, cand=None, kl=None, ws=None) == _lib.KLD_OK
    st = lib.kld_full_vocab_split(A16, A16, _lib.KLD_BF16, 4, 64, 64, 64, None, A16, None, None,
                                  None, None, A16, 1 << 20, None, None, -1)
    assert st == _lib.KLD_ERR_INVALID_ARG
    assert lib.kld_full_vocab_workspace_size(0) > 0
    assert lib.kld_full_vocab_workspace_size(1000) > lib.kld_full_vocab_workspace_size(10)


def tk(lib, **kw):
    a = dict(ri=A16, rl=A16 + 4096, ci=A16 + 8192, cl=A16 + 12288, n=3, k=64, V=1000, kl=A16 + 16384,
             t1=None, nm=None, st=None)
    a.update(kw)
    return lib.kld_topk_tail(a["ri"], a["rl"], a["ci"], a["cl"], a["n"], a["k"], a["V"], a["kl"],
                             a["t1"], a["nm"], a["st"], None)


def test_topk_validation(lib):
    assert tk(lib, k=0) == _lib.KLD_ERR_INVALID_ARG
    assert tk(lib, k=65) == _lib.KLD_ERR_INVALID_ARG
    assert tk(lib, V=64) == _lib.KLD_ERR_INVALID_ARG              # vocab must exceed k
    assert tk(lib, V=1 << 25) == _lib.KLD_ERR_INVALID_ARG
    assert tk(lib, n=-3) == _lib.KLD_ERR_INVALID_ARG
    assert tk(lib, ci=None) == _lib.KLD_ERR_INVALID_ARG
    assert tk(lib, ri=A16 + 2) == _lib.KLD_ERR_ALIGNMENT
    assert tk(lib, rl=A16 + 1) == _lib.KLD_ERR_ALIGNMENT
    assert tk(lib, n=0) == _lib.KLD_OK


def rd(lib, **kw):
    a = dict(kl=A16, ra=None, ca=None, t1=None, lr=None, lc=None, m=None, n=100, q=(0.5,), t=(),
             out=A16 + 4096, ws=A16 + 65536, wsb=None, st=None)
    a.update(kw)
    qs = (ctypes.c_double * max(8, len(a["q"])))(*a["q"])
    ts = (ctypes.c_float * 8)(*a["t"])
    wsb = lib.kld_reduce_workspace_size(a["n"]) if a["wsb"] is None else a["wsb"]
    return lib.kld_reduce_stats(a["kl"], a["ra"], a["ca"], a["t1"], a["lr"], a["lc"], a["m"], a["n"],
                                ctypes.cast(qs, ctypes.c_void_p), len(a["q"]),
                                ctypes.cast(ts, ctypes.c_void_p), len(a["t"]), a["out"], a["ws"], wsb,
                                a["st"], None)


def test_reduce_validation(lib):
    assert rd(lib, q=(1.5,)) == _lib.KLD_ERR_INVALID_ARG
    assert rd(lib, q=(-0.1,)) == _lib.KLD_ERR_INVALID_ARG
    assert rd(lib, q=tuple([0.5] * 9)) == _lib.KLD_ERR_INVALID_ARG
    assert rd(lib, ra=A16) == _lib.KLD_ERR_INVALID_ARG            # argmax pair incomplete
    assert rd(lib, out=None) == _lib.KLD_ERR_INVALID_ARG
    assert rd(lib, n=-1) == _lib.KLD_ERR_INVALID_ARG
    assert rd(lib, ws=None) == _lib.KLD_ERR_WORKSPACE
    assert rd(lib, wsb=16) == _lib.KLD_ERR_WORKSPACE
    assert rd(lib, ws=A16 + 128) == _lib.KLD_ERR_ALIGNMENT
    assert rd(lib, out=A16 + 4) == _lib.KLD_ERR_ALIGNMENT


def sr(lib, **kw):
    a = dict(cand=A16, dtype=_lib.KLD_BF16, n=4, V=4096, ld=4096, top=A16 + 65536, k=512, rows=None, tgt=None,
             kl=A16 + 131072, am=None, t1=None, lpc=None, lpr=None, ws=A16 + (1 << 19), wsb=None, st=None)
    a.update(kw)
    wsb = lib.kld_sparse_ref_workspace_size(max(a["n"], 0), max(a["k"], 1)) if a["wsb"] is None else a["wsb"]
    return lib.kld_sparse_ref_score(a["cand"], a["dtype"], a["n"], a["V"], a["ld"], a["top"], a["k"], a["rows"],
                                    a["tgt"], a["kl"], a["am"], a["t1"], a["lpc"], a["lpr"], a["ws"], wsb,
                                    a["st"], None)


def test_sparse_ref_validation(lib):
    assert sr(lib, dtype=3) == _lib.KLD_ERR_UNSUPPORTED
    assert sr(lib, k=0) == _lib.KLD_ERR_INVALID_ARG
    assert sr(lib, k=_lib.KLD_SPARSE_MAX_K + 1) == _lib.KLD_ERR_INVALID_ARG
    assert sr(lib, k=100, V=64, ld=64) == _lib.KLD_ERR_INVALID_ARG       # more listed ids than the vocabulary
    assert sr(lib, V=(1 << 22) + 8, ld=(1 << 22) + 8) == _lib.KLD_ERR_UNSUPPORTED
    assert sr(lib, ld=4000) == _lib.KLD_ERR_INVALID_ARG
    assert sr(lib, n=-1) == _lib.KLD_ERR_INVALID_ARG
    assert sr(lib, lpc=A16) == _lib.KLD_ERR_INVALID_ARG                  # target lp without targets
    assert sr(lib, lpr=A16) == _lib.KLD_ERR_INVALID_ARG                  # reference lp without its rows
    assert sr(lib, top=None) == _lib.KLD_ERR_INVALID_ARG
    assert sr(lib, kl=None) == _lib.KLD_ERR_INVALID_ARG
    assert sr(lib, ws=None) == _lib.KLD_ERR_WORKSPACE
    assert sr(lib, wsb=1024) == _lib.KLD_ERR_WORKSPACE
    assert sr(lib, cand=MIS) == _lib.KLD_ERR_ALIGNMENT
    assert sr(lib, ld=4100) == _lib.KLD_ERR_ALIGNMENT                    # 8200-byte rows
    assert sr(lib, top=A16 + 4) == _lib.KLD_ERR_ALIGNMENT
    assert sr(lib, ws=A16 + 64) == _lib.KLD_ERR_ALIGNMENT
    assert sr(lib, n=0) == _lib.KLD_OK
    assert lib.kld_sparse_ref_workspace_size(10, 512) > lib.kld_sparse_ref_workspace_size(10, 64)
    assert lib.kld_sparse_ref_workspace_size(10, 0) == 0


def cp(lib, **kw):
    a = dict(x=A16, dtype=_lib.KLD_BF16, n=4, V=4096, ld=4096, k=512, tgt=None, top=A16 + 65536,
             rows=A16 + 131072, ws=A16 + (1 << 19), wsb=None, st=None)
    a.update(kw)
    wsb = lib.kld_sparse_capture_workspace_size(max(a["n"], 0), max(a["k"], 1)) if a["wsb"] is None else a["wsb"]
    return lib.kld_sparse_capture(a["x"], a["dtype"], a["n"], a["V"], a["ld"], a["k"], a["tgt"], a["top"],
                                  a["rows"], a["ws"], wsb, a["st"], None)


def test_sparse_capture_validation(lib):
    assert cp(lib, dtype=2) == _lib.KLD_ERR_UNSUPPORTED
    assert cp(lib, k=0) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, k=_lib.KLD_SPARSE_MAX_K + 1) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, k=65, V=64, ld=64) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, V=(1 << 22) + 8, ld=(1 << 22) + 8) == _lib.KLD_ERR_UNSUPPORTED
    assert cp(lib, ld=4000) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, n=-2) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, top=None) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, rows=None) == _lib.KLD_ERR_INVALID_ARG
    assert cp(lib, ws=None) == _lib.KLD_ERR_WORKSPACE
    assert cp(lib, wsb=4096) == _lib.KLD_ERR_WORKSPACE
    assert cp(lib, x=MIS) == _lib.KLD_ERR_ALIGNMENT
    assert cp(lib, ld=4100) == _lib.KLD_ERR_ALIGNMENT
    assert cp(lib, top=A16 + 4) == _lib.KLD_ERR_ALIGNMENT
    assert cp(lib, ws=A16 + 32) == _lib.KLD_ERR_ALIGNMENT
    assert cp(lib, n=0) == _lib.KLD_OK
    assert lib.kld_sparse_capture_workspace_size(2, 64) > _lib.KLD_CAPTURE_CANDIDATES * 8


def sh(lib, **kw):
    a = dict(step=1, ns=2, g=A16, b=A16 + 65536, kl=A16 + 131072, n=100, q=(0.5,), out=None,
             ws=A16 + (1 << 19), wsb=None)
    a.update(kw)
    qs = (ctypes.c_double * max(8, len(a["q"])))(*a["q"])
    ts = (ctypes.c_float * 8)()
    wsb = lib.kld_reduce_shard_workspace_size(max(a["n"], 0)) if a["wsb"] is None else a["wsb"]
    return lib.kld_reduce_shard_step(a["step"], a["ns"], a["g"], a["b"], a["kl"], None, None, None, None, None,
                                     None, a["n"], ctypes.cast(qs, ctypes.c_void_p), len(a["q"]),
                                     ctypes.cast(ts, ctypes.c_void_p), 0, a["out"], a["ws"], wsb, None, None)


def test_reduce_shard_validation(lib):
    last = _lib.KLD_SHARD_STEPS - 1
    assert sh(lib, step=-1) == _lib.KLD_ERR_INVALID_ARG
    assert sh(lib, step=last + 1) == _lib.KLD_ERR_INVALID_ARG
    assert sh(lib, ns=0) == _lib.KLD_ERR_INVALID_ARG
    assert sh(lib, g=None) == _lib.KLD_ERR_INVALID_ARG                 # the previous blocks are needed
    assert sh(lib, b=None) == _lib.KLD_ERR_INVALID_ARG                 # this shard's block is needed
    assert sh(lib, step=last, b=None, out=None) == _lib.KLD_ERR_INVALID_ARG
    assert sh(lib, q=(2.0,)) == _lib.KLD_ERR_INVALID_ARG
    assert sh(lib, kl=None) == _lib.KLD_ERR_INVALID_ARG
    assert sh(lib, ws=None) == _lib.KLD_ERR_WORKSPACE
    assert sh(lib, wsb=8) == _lib.KLD_ERR_WORKSPACE
    assert sh(lib, g=A16 + 8) == _lib.KLD_ERR_ALIGNMENT
    assert sh(lib, ws=A16 + 64) == _lib.KLD_ERR_ALIGNMENT
    assert sh(lib, step=last, b=None, out=A16 + 4) == _lib.KLD_ERR_ALIGNMENT
    assert lib.kld_reduce_shard_block_bytes() >= 16 * 256 * 4
    assert lib.kld_reduce_shard_workspace_size(10) >= 4 * 16 * 256 * 4   # the four passes' all-shard histograms


def test_paired_struct_size_matches_header():
    assert ctypes.sizeof(_lib.KldPaired) == 144


def pc(lib, **kw):
    a = dict(a=A16, b=A16 + 4096, mask=None, n=4, L=16, cl=A16 + 8192, C=3, rs=A16 + 12288, B=5,
             q=(0.025, 0.975), out=A16 + 16384, boot=None, ws=A16 + 65536, wsb=None, st=None)
    a.update(kw)
    wsb = lib.kld_paired_workspace_size(max(a["n"], 0), max(a["C"], 0), max(a["B"], 0)) if a["wsb"] is None \
        else a["wsb"]
    qs = (ctypes.c_double * max(len(a["q"]), 1))(*a["q"])
    return lib.kld_paired_compare(a["a"], a["b"], a["mask"], a["n"], a["L"], a["cl"], a["C"], a["rs"], a["B"],
                                  ctypes.cast(qs, ctypes.c_void_p), len(a["q"]), a["out"], a["boot"], a["ws"],
                                  wsb, a["st"], None)


def test_paired_validation(lib):
    assert pc(lib, n=-1) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, L=0) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, C=0) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, B=-1) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, B=1 << 19, C=1 << 12) == _lib.KLD_ERR_INVALID_ARG        # draws beyond 2^31
    assert pc(lib, q=(1.5,)) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, q=(0.5,) * 9) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, a=None) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, cl=None) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, rs=None) == _lib.KLD_ERR_INVALID_ARG                     # draws needed when B > 0
    assert pc(lib, out=None) == _lib.KLD_ERR_INVALID_ARG
    assert pc(lib, ws=None) == _lib.KLD_ERR_WORKSPACE
    assert pc(lib, wsb=8) == _lib.KLD_ERR_WORKSPACE
    assert pc(lib, ws=A16 + 64) == _lib.KLD_ERR_ALIGNMENT
    assert pc(lib, out=A16 + 4) == _lib.KLD_ERR_ALIGNMENT
    assert pc(lib, a=MIS) == _lib.KLD_ERR_ALIGNMENT                          # rows are read as 16-byte vectors
    assert pc(lib, b=A16 + 4104) == _lib.KLD_ERR_ALIGNMENT
    assert pc(lib, boot=A16 + 4) == _lib.KLD_ERR_ALIGNMENT
    small = lib.kld_paired_workspace_size(10, 3, 5)
    assert lib.kld_paired_workspace_size(1000, 3, 5) > small
    assert lib.kld_paired_workspace_size(10, 3, 5000) > small
