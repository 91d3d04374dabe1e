"""Parity oracle for combined sparse decode attention (TEST INFRASTRUCTURE).

A thin ctypes/numpy wrapper around ``csa_oracle.c``: a plain fp64 CPU
definition of one decode step of combined sparse attention -- pinned prefix,
sliding window and Quest-style top-k pages -- over a paged GQA KV cache
("Accelerating Long-Context Decoding in Large-Scale Hybrid LLMs Without
Retraining", abstract; Quest named in the arxivlens analysis, "Methodology";
paged top-k and full-size cache in the roboaidigest post, "The Move" and
"Why It Matters").

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library and never imports it; inputs reach both sides from the seeded
generators in ``long_context_decoding_b200.workloads``.

bf16 tensors are passed as ``numpy.uint16`` arrays holding the raw bits.

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle.py`` (brute force, closed forms, invariants and library
routines); see the header of ``csa_oracle.c`` for the readings it takes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "libcsa_oracle.so")
_lib = None


@dataclass(frozen=True)
class Dims:
    """Problem shape: batch, query heads, kv heads, head dim, page size,
    logical pages per sequence (page-table row length), physical pages."""

    B: int
    Hq: int
    Hkv: int
    D: int
    ps: int
    max_pages: int
    num_pages: int

    def arr(self):
        return (ctypes.c_int * 7)(self.B, self.Hq, self.Hkv, self.D, self.ps,
                                  self.max_pages, self.num_pages)


def build(force: bool = False) -> str:
    """Compile csa_oracle.c into libcsa_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_meta.argtypes = [P, P, P, P, P]
        lib.oracle_scores.argtypes = [P, P, P, P, P, I, I, P]
        lib.oracle_select.argtypes = [P, P, P, I, I, I, I, P, P]
        lib.oracle_token_mask.argtypes = [P, P, I, I, P, P, I, I, P]
        lib.oracle_attend.argtypes = [P, P, P, P, P, P, I, I, P, P, I, I, ctypes.c_double, P, P]
        lib.oracle_meta_fp8.argtypes = [P, P, P, P, P]
        lib.oracle_scores_fp8.argtypes = [P, P, P, P, P, I, I, P]
        lib.oracle_fp8_round.argtypes = [ctypes.c_double, I]
        lib.oracle_fp8_round.restype = ctypes.c_double
        lib.oracle_fp8_encode.argtypes = [ctypes.c_double]
        lib.oracle_fp8_decode.argtypes = [I]
        lib.oracle_fp8_decode.restype = ctypes.c_double
        lib.oracle_fp8_row_exponent.argtypes = [ctypes.c_double]
        for f in (lib.oracle_set_threads, lib.oracle_meta, lib.oracle_scores, lib.oracle_select,
                  lib.oracle_token_mask, lib.oracle_attend, lib.oracle_meta_fp8,
                  lib.oracle_scores_fp8, lib.oracle_fp8_encode, lib.oracle_fp8_row_exponent):
            f.restype = I
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid argument (rc={rc})")


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (n <= 0 leaves it); returns the count in use."""
    return int(_load().oracle_set_threads(int(n)))


def meta(d: Dims, k_cache, page_table, seq_lens, meta_init=None):
    """Per (physical page, kv-head, channel) min and max key over valid tokens.

    Returns uint16 [num_pages][Hkv][2][D]; pages not reached keep ``meta_init``
    (zeros when not given)."""
    lib = _load()
    out = np.zeros((d.num_pages, d.Hkv, 2, d.D), np.uint16) if meta_init is None \
        else np.array(meta_init, dtype=np.uint16, copy=True)
    k, kp = _c(k_cache, np.uint16)
    pt, ptp = _c(page_table, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    _check(lib.oracle_meta(d.arr(), kp, ptp, slp, out.ctypes.data_as(ctypes.c_void_p)), "meta")
    return out


def scores(d: Dims, q, k_cache, page_table, seq_lens, prefix: int, window: int):
    """Quest upper-bound scores, float64 [B][Hkv][max_pages]; NaN off the candidates."""
    lib = _load()
    out = np.empty((d.B, d.Hkv, d.max_pages), np.float64)
    qq, qp = _c(q, np.uint16)
    k, kp = _c(k_cache, np.uint16)
    pt, ptp = _c(page_table, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    _check(lib.oracle_scores(d.arr(), qp, kp, ptp, slp, int(prefix), int(window),
                             out.ctypes.data_as(ctypes.c_void_p)), "scores")
    return out


def select(d: Dims, score, seq_lens, prefix: int, window: int, budget: int, max_sel: int):
    """Top-k candidate pages (score desc, then page asc), returned ascending.

    Returns (sel int32 [B][Hkv][max_sel], nsel int32 [B][Hkv]); unused slots = -1."""
    lib = _load()
    sel = np.full((d.B, d.Hkv, max(max_sel, 1)), -1, np.int32)
    nsel = np.zeros((d.B, d.Hkv), np.int32)
    sc, scp = _c(score, np.float64)
    sl, slp = _c(seq_lens, np.int32)
    _check(lib.oracle_select(d.arr(), scp, slp, int(prefix), int(window), int(budget),
                             int(max_sel), sel.ctypes.data_as(ctypes.c_void_p),
                             nsel.ctypes.data_as(ctypes.c_void_p)), "select")
    return sel[:, :, :max_sel], nsel


def token_mask(d: Dims, seq_lens, prefix: int, window: int, sel, nsel, max_sel: int,
               dense: bool = False):
    """Attended-token mask, uint8 [B][Hkv][max_pages * ps]."""
    lib = _load()
    m = np.zeros((d.B, d.Hkv, d.max_pages * d.ps), np.uint8)
    sl, slp = _c(seq_lens, np.int32)
    s, sp = _c(sel if sel is not None else np.zeros((d.B, d.Hkv, 1), np.int32), np.int32)
    n, npp = _c(nsel if nsel is not None else np.zeros((d.B, d.Hkv), np.int32), np.int32)
    _check(lib.oracle_token_mask(d.arr(), slp, int(prefix), int(window), sp, npp, int(max_sel),
                                 int(bool(dense)), m.ctypes.data_as(ctypes.c_void_p)), "token_mask")
    return m


def attend(d: Dims, q, k_cache, v_cache, page_table, seq_lens, prefix: int, window: int,
           sel, nsel, max_sel: int, scale: float, dense: bool = False):
    """Softmax attention over the attended set (or every valid token when dense).

    Returns (out float64 [B][Hq][D], lse float64 [B][Hq])."""
    lib = _load()
    out = np.empty((d.B, d.Hq, d.D), np.float64)
    lse = np.empty((d.B, d.Hq), np.float64)
    qq, qp = _c(q, np.uint16)
    k, kp = _c(k_cache, np.uint16)
    v, vp = _c(v_cache, np.uint16)
    pt, ptp = _c(page_table, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    if sel is None:
        sel = np.zeros((d.B, d.Hkv, max(max_sel, 1)), np.int32)
        nsel = np.zeros((d.B, d.Hkv), np.int32)
    s, sp = _c(sel, np.int32)
    n, npp = _c(nsel, np.int32)
    _check(lib.oracle_attend(d.arr(), qp, kp, vp, ptp, slp, int(prefix), int(window), sp, npp,
                             int(max_sel), int(bool(dense)), float(scale),
                             out.ctypes.data_as(ctypes.c_void_p),
                             lse.ctypes.data_as(ctypes.c_void_p)), "attend")
    return out, lse


def step(d: Dims, q, k_cache, v_cache, page_table, seq_lens, prefix: int, window: int,
         budget: int, max_sel: int, scale: float):
    """One sparse decode step: scores -> top-k -> attention.  Returns a dict."""
    sc = scores(d, q, k_cache, page_table, seq_lens, prefix, window)
    sel, nsel = select(d, sc, seq_lens, prefix, window, budget, max_sel)
    out, lse = attend(d, q, k_cache, v_cache, page_table, seq_lens, prefix, window, sel, nsel,
                      max_sel, scale)
    return {"scores": sc, "sel": sel, "nsel": nsel, "out": out, "lse": lse}


# ---------------------------------------------------------------- fp8 metadata
# An optional lower-precision copy of the metadata (not a step of the pages'
# method): per (physical page, kv-head) 2*D bytes of E4M3 -- min rounded down,
# max rounded up after scaling by 2^-e -- and a 16-byte trailer holding e
# (int32) and zeros.  See csa_oracle.c for the definition.
def meta8_row_bytes(D: int) -> int:
    return 2 * D + 16


def fp8_round(y: float, up: bool) -> float:
    """Largest (up=False) / smallest (up=True) E4M3 value <= / >= y (|y| <= 448)."""
    return float(_load().oracle_fp8_round(float(y), 1 if up else 0))


def fp8_encode(v: float) -> int:
    return int(_load().oracle_fp8_encode(float(v)))


def fp8_decode(x: int) -> float:
    return float(_load().oracle_fp8_decode(int(x)))


def fp8_row_exponent(a: float) -> int:
    """Smallest e with a * 2^-e <= 448 (0 for a = 0)."""
    return int(_load().oracle_fp8_row_exponent(float(a)))


def meta_fp8(d: Dims, meta_bf16, page_table, seq_lens, meta8_init=None):
    """fp8 copy of the (exact, bf16) metadata of every page reached by a valid
    token.  Returns uint8 [num_pages][Hkv][2*D + 16]."""
    lib = _load()
    shape = (d.num_pages, d.Hkv, meta8_row_bytes(d.D))
    out = np.zeros(shape, np.uint8) if meta8_init is None \
        else np.array(meta8_init, dtype=np.uint8, copy=True)
    m, mp = _c(meta_bf16, np.uint16)
    pt, ptp = _c(page_table, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    _check(lib.oracle_meta_fp8(d.arr(), mp, ptp, slp, out.ctypes.data_as(ctypes.c_void_p)),
           "meta_fp8")
    return out


def scores_fp8(d: Dims, q, meta8, page_table, seq_lens, prefix: int, window: int):
    """Quest scores from the fp8 metadata, float64 [B][Hkv][max_pages]; NaN off
    the candidates."""
    lib = _load()
    out = np.empty((d.B, d.Hkv, d.max_pages), np.float64)
    qq, qp = _c(q, np.uint16)
    m8, m8p = _c(meta8, np.uint8)
    pt, ptp = _c(page_table, np.int32)
    sl, slp = _c(seq_lens, np.int32)
    _check(lib.oracle_scores_fp8(d.arr(), qp, m8p, ptp, slp, int(prefix), int(window),
                                 out.ctypes.data_as(ctypes.c_void_p)), "scores_fp8")
    return out


def step_fp8(d: Dims, q, k_cache, v_cache, page_table, seq_lens, prefix: int, window: int,
             budget: int, max_sel: int, scale: float):
    """One sparse decode step scored on the fp8 metadata (derived from the
    exact metadata of the cache): scores -> top-k -> attention."""
    m = meta(d, k_cache, page_table, seq_lens)
    m8 = meta_fp8(d, m, page_table, seq_lens)
    sc = scores_fp8(d, q, m8, page_table, seq_lens, prefix, window)
    sel, nsel = select(d, sc, seq_lens, prefix, window, budget, max_sel)
    out, lse = attend(d, q, k_cache, v_cache, page_table, seq_lens, prefix, window, sel, nsel,
                      max_sel, scale)
    return {"meta8": m8, "scores": sc, "sel": sel, "nsel": nsel, "out": out, "lse": lse}
