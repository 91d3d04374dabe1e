"""Pins for the CPU oracle (no GPU): brute force, closed forms, invariants and
library routines, each independent of the oracle's own code.

What each plausible oracle mistake trips:
  * min/max over the wrong slots or tokens  -> test_meta_* (numpy reductions)
  * a dropped min term / wrong sign in the Quest bound -> test_score_box_corners
    (max of q.k over the key box, by enumerating its corners) and the upper
    bound / tightness tests
  * wrong kv-head of a query head, or sum instead of max over the group
    -> test_score_box_corners (per-head scores differ across the group)
  * wrong candidate pages -> test_candidates_brute_force
  * wrong tie rule or order of the selection -> test_select_* (subset
    enumeration and duplicated pages)
  * wrong attended set, softmax, scale or lse -> test_attend_* (torch SDPA in
    fp64 with a mask built from sets of token indices, scipy logsumexp,
    closed forms, page-permutation invariance)
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import workloads as wl

PS = 16


def case_np(B=2, Hq=4, Hkv=2, D=16, lens=(70, 45), seed=0, spare=2, poison=True):
    """Small random paged case on the host (numpy uint16 bf16 bits)."""
    w = wl.Workload("t", B=B, Hq=Hq, Hkv=Hkv, D=D, seq_lens=tuple(lens), prefix=0,
                    window=0, budget=0, seed=seed, spare_pages=spare)
    c = wl.make_case(w, "cpu", poison=poison)
    d = oracle.Dims(B, Hq, Hkv, D, PS, w.max_pages, w.num_pages)
    return d, c, dict(q=wl.bits(c.q), k=wl.bits(c.k_cache), v=wl.bits(c.v_cache),
                      pt=c.page_table.numpy(), sl=c.seq_lens.numpy())


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def token_keys(d, a, b, g):
    """Keys of sequence b, kv-head g in logical token order (float64 [L][D])."""
    L = int(a["sl"][b])
    rows = []
    for t in range(L):
        phys = a["pt"][b, t // PS]
        rows.append(f64(a["k"][phys, g, t % PS]))
    return np.array(rows).reshape(L, d.D)


def token_vals(d, a, b, g):
    L = int(a["sl"][b])
    return np.array([f64(a["v"][a["pt"][b, t // PS], g, t % PS]) for t in range(L)]).reshape(L, d.D)


# ------------------------------------------------------------------ metadata
def test_meta_matches_numpy_reductions():
    d, c, a = case_np(lens=(70, 45, 16, 1), B=4)
    meta = oracle.meta(d, a["k"], a["pt"], a["sl"])
    for b in range(d.B):
        for g in range(d.Hkv):
            keys = token_keys(d, a, b, g)
            L = keys.shape[0]
            for p in range(-(-L // PS)):
                blk = keys[p * PS:min(L, (p + 1) * PS)]
                phys = a["pt"][b, p]
                np.testing.assert_array_equal(f64(meta[phys, g, 0]), blk.min(0))
                np.testing.assert_array_equal(f64(meta[phys, g, 1]), blk.max(0))


def test_meta_single_token_page_is_the_key():
    d, c, a = case_np(lens=(33,), B=1)        # page 2 holds one token
    meta = oracle.meta(d, a["k"], a["pt"], a["sl"])
    phys = a["pt"][0, 2]
    for g in range(d.Hkv):
        np.testing.assert_array_equal(meta[phys, g, 0], a["k"][phys, g, 0])
        np.testing.assert_array_equal(meta[phys, g, 1], a["k"][phys, g, 0])


def test_meta_ignores_poisoned_slots():
    d, c, a = case_np(lens=(21, 40), B=2)      # partial last pages, NaN beyond
    meta = oracle.meta(d, a["k"], a["pt"], a["sl"])
    for b in range(d.B):
        for p in range(-(-int(a["sl"][b]) // PS)):
            assert np.isfinite(f64(meta[a["pt"][b, p]])).all()


def test_meta_and_scores_ignore_finite_garbage_beyond_length():
    """Slots at or past seq_len hold large finite keys (not NaN, which no
    comparison would pick); neither min/max nor the page bound may see them."""
    d, c, a = case_np(lens=(21, 40), B=2, Hq=4, Hkv=2)
    k = a["k"].copy()
    for b, L in enumerate((21, 40)):
        phys = a["pt"][b, L // PS]
        k[phys, :, L % PS:, ::2] = 0x4580          # +4096
        k[phys, :, L % PS:, 1::2] = 0xC580         # -4096
    meta = oracle.meta(d, k, a["pt"], a["sl"])
    sc = oracle.scores(d, a["q"], k, a["pt"], a["sl"], 0, 0)
    a2 = dict(a, k=k)
    G = d.Hq // d.Hkv
    for b, L in enumerate((21, 40)):
        p = L // PS
        for g in range(d.Hkv):
            blk = token_keys(d, a2, b, g)[p * PS:L]
            np.testing.assert_array_equal(f64(meta[a["pt"][b, p], g, 0]), blk.min(0))
            np.testing.assert_array_equal(f64(meta[a["pt"][b, p], g, 1]), blk.max(0))
            assert abs(sc[b, g, p]) < 1000


# -------------------------------------------------------------------- scores
def candidates_brute(L, P, W):
    """Pages holding at least one token t with P' <= t < L - W' (token sets)."""
    Pe, We = min(P, L), min(W, L)
    mid = set(range(Pe, L - We)) if Pe < L - We else set()
    return sorted({t // PS for t in mid})


@pytest.mark.parametrize("L,P,W", [(70, 0, 0), (70, 5, 7), (70, 16, 16), (70, 3, 60),
                                   (70, 40, 40), (70, 100, 0), (1, 0, 0), (33, 17, 0),
                                   (64, 0, 48), (45, 15, 15)])
def test_candidates_brute_force(L, P, W):
    d, c, a = case_np(lens=(L,), B=1, Hq=2, Hkv=1)
    sc = oracle.scores(d, a["q"], a["k"], a["pt"], a["sl"], P, W)
    got = [p for p in range(d.max_pages) if not math.isnan(sc[0, 0, p])]
    assert got == candidates_brute(L, P, W)


def test_score_box_corners():
    """The Quest bound of a head is the max of q.k over the key box
    [min, max]^D, attained at a corner; enumerate all 2^D corners (D = 8).
    The kv-head score is the max of that over the group's query heads."""
    d, c, a = case_np(B=2, Hq=6, Hkv=3, D=8, lens=(50, 37))
    sc = oracle.scores(d, a["q"], a["k"], a["pt"], a["sl"], 0, 0)
    corners = np.array(list(itertools.product((0, 1), repeat=d.D)), dtype=bool)
    G = d.Hq // d.Hkv
    for b in range(d.B):
        for g in range(d.Hkv):
            keys = token_keys(d, a, b, g)
            for p in range(-(-keys.shape[0] // PS)):
                blk = keys[p * PS:(p + 1) * PS]
                lo, hi = blk.min(0), blk.max(0)
                box = np.where(corners, hi, lo)               # [2^D][D]
                best = max((box @ f64(a["q"][b, g * G + j])).max() for j in range(G))
                assert sc[b, g, p] == pytest.approx(best, rel=1e-12, abs=1e-12)


def test_score_upper_bounds_every_head_and_is_tight_for_one_token():
    d, c, a = case_np(B=1, Hq=8, Hkv=2, D=32, lens=(97,))    # last page: 1 token
    sc = oracle.scores(d, a["q"], a["k"], a["pt"], a["sl"], 0, 0)
    G = d.Hq // d.Hkv
    for g in range(d.Hkv):
        keys = token_keys(d, a, 0, g)
        for p in range(-(-97 // PS)):
            blk = keys[p * PS:(p + 1) * PS]
            true_max = max((blk @ f64(a["q"][0, g * G + j])).max() for j in range(G))
            assert sc[0, g, p] >= true_max - 1e-12 * abs(true_max)
        # page 6 holds only token 96: the bound equals max_h q_h.k exactly
        exact = max(float(keys[96] @ f64(a["q"][0, g * G + j])) for j in range(G))
        assert sc[0, g, 6] == pytest.approx(exact, rel=1e-14, abs=1e-14)


def test_score_rewrite_identity():
    """max(a*M, a*m) == max(a,0)*M + min(a,0)*m whenever m <= M (the
    tensor-core form the CUDA scorer evaluates)."""
    rng = np.random.default_rng(0)
    a = rng.standard_normal(100000)
    m = rng.standard_normal(100000)
    M = m + np.abs(rng.standard_normal(100000))
    lhs = np.maximum(a * M, a * m)
    rhs = np.maximum(a, 0) * M + np.minimum(a, 0) * m
    np.testing.assert_array_equal(lhs, rhs)


# ----------------------------------------------------------------- selection
def brute_topk(scores, k):
    """Max-sum subset of size k; among equal sums the lexicographically
    smallest ascending index tuple."""
    n = len(scores)
    best = None
    for comb in itertools.combinations(range(n), k):
        s = sum(scores[i] for i in comb)
        if best is None or s > best[0] or (s == best[0] and comb < best[1]):
            best = (s, comb)
    return list(best[1]) if best else []


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_subset_enumeration(seed):
    rng = np.random.default_rng(seed)
    L = 16 * 12
    d = oracle.Dims(1, 1, 1, 16, PS, 12, 12)
    for kpages in range(0, 13):
        sc = np.full((1, 1, 12), np.nan)
        sc[0, 0, :] = rng.integers(0, 4, 12).astype(float)   # many ties
        sel, nsel = oracle.select(d, sc, np.array([L], np.int32), 0, 0, kpages * PS, 12)
        assert nsel[0, 0] == kpages
        assert list(sel[0, 0, :kpages]) == brute_topk(list(sc[0, 0]), kpages)


def test_select_respects_candidate_range_and_budget():
    d = oracle.Dims(1, 1, 1, 16, PS, 12, 12)
    sc = np.full((1, 1, 12), np.nan)
    L, P, W = 180, 20, 50          # candidates: pages 1 .. 8
    cand = candidates_brute(L, P, W)
    sc[0, 0, cand] = np.arange(len(cand))[::-1].astype(float)
    sel, nsel = oracle.select(d, sc, np.array([L], np.int32), P, W, 3 * PS + 7, 12)
    assert nsel[0, 0] == 3 and list(sel[0, 0, :3]) == cand[:3]
    sel, nsel = oracle.select(d, sc, np.array([L], np.int32), P, W, 100 * PS, 100)
    assert nsel[0, 0] == len(cand) and list(sel[0, 0, :len(cand)]) == cand
    sel, nsel = oracle.select(d, sc, np.array([L], np.int32), P, W, 15, 12)
    assert nsel[0, 0] == 0


def test_select_tie_rule_on_duplicated_pages():
    """Pages with identical keys score identically; the lower page wins."""
    d, c, a = case_np(B=1, Hq=2, Hkv=1, D=16, lens=(16 * 10,))
    k = a["k"].copy()
    src = a["pt"][0, 2]
    for p in (4, 7, 8):
        k[a["pt"][0, p]] = k[src]
    k[src, 0, 0, 0] = 0x4500      # make page 2 the clear winner (k = 2048)
    sc = oracle.scores(d, a["q"], k, a["pt"], a["sl"], 0, 0)
    assert sc[0, 0, 4] == sc[0, 0, 7] == sc[0, 0, 8]
    order = sorted(range(10), key=lambda p: -sc[0, 0, p])
    k_pages = order.index(4) + 2         # take page 4 and exactly one more of the tie
    sel, nsel = oracle.select(d, sc, a["sl"], 0, 0, k_pages * PS, 10)
    chosen = set(sel[0, 0, :nsel[0, 0]])
    assert 4 in chosen and 7 in chosen and 8 not in chosen


# ----------------------------------------------------------------- attention
def attended_tokens(L, P, W, sel):
    Pe, We = min(P, L), min(W, L)
    A = set(range(Pe)) | set(range(L - We, L))
    for p in sel:
        A |= {t for t in range(p * PS, (p + 1) * PS) if t < L}
    return sorted(A)


def sdpa_ref(q, K, V, tokens, scale):
    """torch SDPA in fp64 over the given token indices (one query head)."""
    qt = torch.tensor(q).view(1, 1, 1, -1)
    kt = torch.tensor(K).view(1, 1, K.shape[0], -1)
    vt = torch.tensor(V).view(1, 1, V.shape[0], -1)
    mask = torch.zeros(1, 1, 1, K.shape[0], dtype=torch.bool)
    mask[..., tokens] = True
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.view(-1).numpy()


@pytest.mark.parametrize("P,W,budget", [(5, 7, 32), (16, 16, 0), (0, 0, 48), (3, 9, 160),
                                        (40, 40, 16), (0, 1, 0)])
def test_attend_matches_sdpa_on_token_sets(P, W, budget):
    d, c, a = case_np(B=2, Hq=4, Hkv=2, D=16, lens=(70, 45))
    scale = 1 / math.sqrt(d.D)
    max_sel = 8
    step = oracle.step(d, a["q"], a["k"], a["v"], a["pt"], a["sl"], P, W, budget, max_sel, scale)
    G = d.Hq // d.Hkv
    for b in range(d.B):
        for g in range(d.Hkv):
            K, V = token_keys(d, a, b, g), token_vals(d, a, b, g)
            sel = step["sel"][b, g, :step["nsel"][b, g]]
            toks = attended_tokens(int(a["sl"][b]), P, W, sel)
            for j in range(G):
                h = g * G + j
                ref = sdpa_ref(f64(a["q"][b, h]), K, V, toks, scale)
                np.testing.assert_allclose(step["out"][b, h], ref, rtol=1e-12, atol=1e-13)


def test_attend_dense_equivalence_and_lse():
    from scipy.special import logsumexp
    d, c, a = case_np(B=2, Hq=4, Hkv=2, D=16, lens=(70, 45))
    scale = 0.3
    dense, lse_d = oracle.attend(d, a["q"], a["k"], a["v"], a["pt"], a["sl"], 0, 0, None, None,
                                 1, scale, dense=True)
    # budget >= L and prefix + window >= L both reduce to the dense layer
    for (P, W, budget) in [(0, 0, 10_000), (30, 40, 0), (100, 0, 0)]:
        st = oracle.step(d, a["q"], a["k"], a["v"], a["pt"], a["sl"], P, W, budget, 8, scale)
        np.testing.assert_allclose(st["out"], dense, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(st["lse"], lse_d, rtol=1e-13)
    G = d.Hq // d.Hkv
    for b in range(d.B):
        for h in range(d.Hq):
            K = token_keys(d, a, b, h // G)
            z = scale * (K @ f64(a["q"][b, h]))
            assert lse_d[b, h] == pytest.approx(logsumexp(z), rel=1e-13)


def test_attend_closed_forms():
    d, c, a = case_np(B=1, Hq=2, Hkv=1, D=16, lens=(40,))
    # one attended token: out = v_0, lse = scale * q.k_0
    out, lse = oracle.attend(d, a["q"], a["k"], a["v"], a["pt"], a["sl"], 1, 0,
                             np.zeros((1, 1, 1), np.int32), np.zeros((1, 1), np.int32), 1, 0.5)
    k0 = f64(a["k"][a["pt"][0, 0], 0, 0])
    v0 = f64(a["v"][a["pt"][0, 0], 0, 0])
    for h in range(2):
        np.testing.assert_array_equal(out[0, h], v0)
        assert lse[0, h] == pytest.approx(0.5 * float(k0 @ f64(a["q"][0, h])), rel=1e-14)
    # identical keys: softmax is uniform, out = mean of V over the set
    k = a["k"].copy()
    for p in range(3):
        k[a["pt"][0, p], 0, :, :] = a["k"][a["pt"][0, 0], 0, 0]
    out, lse = oracle.attend(d, a["q"], k, a["v"], a["pt"], a["sl"], 0, 0, None, None, 1, 0.7,
                             dense=True)
    V = token_vals(d, a, 0, 0)
    np.testing.assert_allclose(out[0, 0], V.mean(0), rtol=1e-12, atol=1e-14)
    # empty sequence: zero output, lse = -inf
    d0 = oracle.Dims(1, 2, 1, 16, PS, d.max_pages, d.num_pages)
    out, lse = oracle.attend(d0, a["q"], a["k"], a["v"], a["pt"], np.zeros(1, np.int32), 0, 0,
                             None, None, 1, 0.5, dense=True)
    assert (out == 0).all() and np.isneginf(lse).all()


def test_attend_invariant_to_physical_page_permutation():
    d, c, a = case_np(B=2, Hq=4, Hkv=2, D=16, lens=(70, 45))
    st = oracle.step(d, a["q"], a["k"], a["v"], a["pt"], a["sl"], 5, 9, 32, 4, 0.25)
    rng = np.random.default_rng(1)
    perm = rng.permutation(d.num_pages)            # new slot of old page i
    k2 = np.empty_like(a["k"]); v2 = np.empty_like(a["v"])
    k2[perm] = a["k"]; v2[perm] = a["v"]
    pt2 = perm[a["pt"]].astype(np.int32)
    st2 = oracle.step(d, a["q"], k2, v2, pt2, a["sl"], 5, 9, 32, 4, 0.25)
    np.testing.assert_array_equal(st["sel"], st2["sel"])
    np.testing.assert_array_equal(st["out"], st2["out"])


def test_oracle_rejects_bad_arguments():
    d, c, a = case_np(B=1, Hq=2, Hkv=1, D=16, lens=(40,))
    bad = a["pt"].copy(); bad[0, 1] = d.num_pages
    with pytest.raises(ValueError):
        oracle.scores(d, a["q"], a["k"], bad, a["sl"], 0, 0)
    with pytest.raises(ValueError):
        oracle.scores(d, a["q"], a["k"], a["pt"], np.array([d.max_pages * PS + 1], np.int32), 0, 0)
