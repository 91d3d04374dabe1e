"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare.

Data flows one way: inputs come from ``workloads`` (copied to the host for
the oracle), oracle outputs may feed the CUDA path (the decode parity runs
the kernels on the oracle's page selection), and no number computed by the
CUDA path is ever given to the oracle.  The one place where the GPU's result
steers what the oracle computes is a tie: where several selections are
correct (pages whose oracle scores lie inside the tie band are
interchangeable), ``oracle_on_valid_choice`` builds the selection from the
oracle's own pages above the band plus the GPU's pick among the band pages,
after ``check_selection`` has shown the pick to be one of the valid ones, and
the oracle attends over that set.  Only page indices the oracle's scores
admit pass; the oracle's arithmetic sees the same inputs as always.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl

PS = 16
# Tolerances on the attention output, against the oracle's fp64 result rounded
# to fp32: bf16 inputs, bf16 output.
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
# Selection: sets must match exactly where the oracle's k-th / (k+1)-th score
# gap exceeds this relative amount; inside the band any choice is valid.
SEL_BAND = 1e-3


class Run:
    """One layer on the GPU plus its host copy for the oracle."""

    def __init__(self, case: wl.Case, prefix=None, window=None, budget=None):
        self.c = case
        w = case.w
        self.prefix = w.prefix if prefix is None else prefix
        self.window = case.window if window is None else window
        self.budget = case.budget if budget is None else budget
        self.max_sel = max(1, max(w.max_sel, self.budget // PS))
        self.d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, self.max_sel)
        self.od = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
        self.ws = csa.new_workspace(self.d, case.q.device)
        self.layer = csa.Layer(self.d, case.k_cache, case.v_cache, case.page_table, case.seq_lens,
                               self.prefix, self.window, self.budget, ws=self.ws)
        self.scale = 1.0 / math.sqrt(w.D)
        self.refresh_host()

    def refresh_host(self):
        c = self.c
        self.h = dict(q=wl.bits(c.q), k=wl.bits(c.k_cache), v=wl.bits(c.v_cache),
                      pt=c.page_table.cpu().numpy(), sl=c.seq_lens.cpu().numpy())

    # ---------------------------------------------------------------- GPU
    def gpu_meta(self):
        self.layer.rebuild_meta()
        return self.layer.meta

    def gpu_select(self, scores=True):
        sc = None
        if scores:
            sc = torch.full((self.d.B, self.d.Hkv, self.d.max_pages_per_seq), float("nan"),
                            dtype=torch.float32, device=self.c.q.device)
        csa.score_select(self.d, self.c.q, self.layer.meta, self.c.page_table, self.c.seq_lens,
                         self.prefix, self.window, self.budget, self.layer.sel,
                         self.layer.n_sel, self.ws, scores_out=sc)
        return sc

    def gpu_decode(self, sel, nsel):
        out = torch.empty((self.d.B, self.d.Hq, self.d.D), dtype=torch.bfloat16,
                          device=self.c.q.device)
        lse = torch.empty((self.d.B, self.d.Hq), dtype=torch.float32, device=self.c.q.device)
        csa.decode(self.d, self.c.q, self.c.k_cache, self.c.v_cache, self.c.page_table,
                   self.c.seq_lens, sel, nsel, self.prefix, self.window, out, self.ws, lse)
        return out, lse

    def gpu_dense(self):
        out = torch.empty((self.d.B, self.d.Hq, self.d.D), dtype=torch.bfloat16,
                          device=self.c.q.device)
        lse = torch.empty((self.d.B, self.d.Hq), dtype=torch.float32, device=self.c.q.device)
        csa.decode_full(self.d, self.c.q, self.c.k_cache, self.c.v_cache, self.c.page_table,
                        self.c.seq_lens, out, self.ws, lse)
        return out, lse

    # ---------------------------------------------------------------- oracle
    def oracle_meta(self):
        return oracle.meta(self.od, self.h["k"], self.h["pt"], self.h["sl"])

    def oracle_step(self):
        st = oracle.step(self.od, self.h["q"], self.h["k"], self.h["v"], self.h["pt"],
                         self.h["sl"], self.prefix, self.window, self.budget, self.max_sel,
                         self.scale)
        return st

    def oracle_dense(self):
        return oracle.attend(self.od, self.h["q"], self.h["k"], self.h["v"], self.h["pt"],
                             self.h["sl"], 0, 0, None, None, 1, self.scale, dense=True)


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_meta_equal(run: Run, gpu_meta: torch.Tensor):
    """Metadata is exact (min/max of bf16 values): compare values over every
    page a sequence owns through a valid token."""
    ref = run.oracle_meta()
    got = wl.bits(gpu_meta)
    sl, pt = run.h["sl"], run.h["pt"]
    for b in range(run.d.B):
        np_b = -(-int(sl[b]) // PS)
        phys = pt[b, :np_b]
        np.testing.assert_array_equal(f64(got[phys]), f64(ref[phys]),
                                      err_msg=f"metadata of sequence {b}")


def assert_scores_close(gpu_scores: torch.Tensor, ref: np.ndarray):
    got = gpu_scores.cpu().numpy().astype(np.float64)
    cand = ~np.isnan(ref)
    assert np.array_equal(~np.isnan(got), cand), "scores written off the candidate pages"
    # fp32 sums of exact bf16 products vs fp64: error ~ D * eps32 * |terms|
    np.testing.assert_allclose(got[cand], ref[cand], rtol=2e-5, atol=2e-3)


def check_selection(gpu_sel, gpu_nsel, ref_scores, ref_sel, ref_nsel, gpu_scores=None):
    """Parity of the page selection with the oracle (band rule), plus the
    validity of the GPU's choice (ascending, unique candidates; exactly the
    top-k of the kernel's own fp32 scores with ties to the lower page)."""
    gs = gpu_sel.cpu().numpy()
    gn = gpu_nsel.cpu().numpy()
    np.testing.assert_array_equal(gn, ref_nsel, err_msg="n_sel")
    own = gpu_scores.cpu().numpy() if gpu_scores is not None else None
    exact_units = 0
    B, Hkv = gn.shape
    for b in range(B):
        for g in range(Hkv):
            k = int(gn[b, g])
            got = gs[b, g, :k]
            sc = ref_scores[b, g]
            cand = np.where(~np.isnan(sc))[0]
            assert np.all(np.diff(got) > 0), "selection not strictly ascending"
            assert np.all(np.isin(got, cand)), "selected a non-candidate page"
            want = ref_sel[b, g, :k]
            if k == 0 or k == len(cand):
                np.testing.assert_array_equal(got, want)
                exact_units += 1
                continue
            order = sorted(cand, key=lambda p: (-sc[p], p))
            s_k, s_k1 = sc[order[k - 1]], sc[order[k]]
            gap = abs(s_k - s_k1) / max(abs(s_k), 1e-30)
            if gap > SEL_BAND:
                np.testing.assert_array_equal(got, want, err_msg=f"unit ({b},{g})")
                exact_units += 1
            else:
                delta = SEL_BAND * abs(s_k)
                must = set(cand[sc[cand] > s_k + delta])
                never = set(cand[sc[cand] < s_k - delta])
                gset = set(got.tolist())
                assert must <= gset, f"unit ({b},{g}) misses a page above the band"
                assert not (never & gset), f"unit ({b},{g}) took a page below the band"
            if own is not None:
                o = own[b, g]
                top = sorted(cand, key=lambda p: (-o[p], p))[:k]
                np.testing.assert_array_equal(got, np.sort(top),
                                              err_msg=f"unit ({b},{g}) is not the top-k of its "
                                                      "own fp32 scores")
    return exact_units


def assert_out_close(out: torch.Tensor, lse: torch.Tensor, ref_out: np.ndarray,
                     ref_lse: np.ndarray, what=""):
    got = out.float().cpu().numpy().astype(np.float64)
    ref = ref_out.astype(np.float32).astype(np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= OUT_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"
    gl = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin), f"{what}: lse finiteness"
    np.testing.assert_allclose(gl[fin], ref_lse[fin], rtol=1e-4, atol=1e-3, err_msg=what)
    return float(err.max()), float(err.mean())


def band_parts(sc: np.ndarray, k: int):
    """Pages of one unit the oracle's scores fix: (must, band), where every
    valid top-k selection holds all of ``must`` and k - len(must) pages of
    ``band`` (the tie band of the k-th score, band rule above)."""
    cand = np.where(~np.isnan(sc))[0]
    if k == 0:
        return set(), set()
    if k >= len(cand):
        return set(cand.tolist()), set()
    order = sorted(cand, key=lambda p: (-sc[p], p))
    s_k, s_k1 = sc[order[k - 1]], sc[order[k]]
    gap = abs(s_k - s_k1) / max(abs(s_k), 1e-30)
    if gap > SEL_BAND:
        return set(int(p) for p in order[:k]), set()
    delta = SEL_BAND * abs(s_k)
    must = set(int(p) for p in cand[sc[cand] > s_k + delta])
    band = set(int(p) for p in cand[np.abs(sc[cand] - s_k) <= delta])
    return must, band


def valid_choice(gpu_sel, gpu_nsel, ref_scores, ref_sel, ref_nsel):
    """Per unit, the selection the oracle attends over to check the GPU's
    output: the oracle's own where the GPU chose it, else the oracle's pages
    above the tie band plus the GPU's pick among the band pages (asserted to
    be a valid top-k first).  Returns (sel int32 [B][Hkv][W], nsel, n_same)."""
    gs = np.asarray(gpu_sel.cpu().numpy() if torch.is_tensor(gpu_sel) else gpu_sel)
    gn = np.asarray(gpu_nsel.cpu().numpy() if torch.is_tensor(gpu_nsel) else gpu_nsel)
    B, Hkv = gn.shape
    width = max(1, ref_sel.shape[2])
    sel = np.full((B, Hkv, width), -1, np.int32)
    nsel = np.asarray(ref_nsel, np.int32).copy()
    same = 0
    for b in range(B):
        for g in range(Hkv):
            k = int(ref_nsel[b, g])
            assert int(gn[b, g]) == k, f"unit ({b},{g}): n_sel"
            want = ref_sel[b, g, :k]
            got = gs[b, g, :k]
            if np.array_equal(got, want):
                sel[b, g, :k] = want
                same += 1
                continue
            must, band = band_parts(ref_scores[b, g], k)
            picked = set(int(p) for p in got.tolist()) & band
            assert must <= set(got.tolist()) and len(must) + len(picked) == k, \
                f"unit ({b},{g}): the GPU's selection is not a valid top-k"
            sel[b, g, :k] = np.array(sorted(must | picked), np.int32)
    return sel, nsel, same


def oracle_on_valid_choice(od, h, prefix, window, scale, gpu_sel, gpu_nsel, ref):
    """The oracle's attention for the GPU's (valid) selection of every unit:
    (out, lse, n_same).  Calls the oracle again only when some unit's
    selection differs from the oracle's own."""
    sel, nsel, same = valid_choice(gpu_sel, gpu_nsel, ref["scores"], ref["sel"], ref["nsel"])
    if same == nsel.size:
        return ref["out"], ref["lse"], same
    out, lse = oracle.attend(od, h["q"], h["k"], h["v"], h["pt"], h["sl"], prefix, window, sel,
                             nsel, sel.shape[2], scale)
    return out, lse, same
