"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs (metadata bit-exact, scores to fp32 accuracy, selection by
the band rule, attention within max-abs 2e-2 / mean-abs 2e-3 of fp32)."""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl
from parity import (Run, assert_meta_equal, assert_out_close, assert_scores_close,
                    check_selection, oracle_on_valid_choice)

pytestmark = pytest.mark.gpu
PS = 16


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(0)
    yield


def full_check(run: Run, dense=True):
    """meta -> score/select -> decode (on the oracle's selection) -> dense."""
    meta = run.gpu_meta()
    assert_meta_equal(run, meta)
    ref = run.oracle_step()
    scores = run.gpu_select()
    torch.cuda.synchronize()
    assert_scores_close(scores, ref["scores"])
    check_selection(run.layer.sel, run.layer.n_sel, ref["scores"], ref["sel"], ref["nsel"],
                    gpu_scores=scores)
    # decode parity on the oracle's own selection (oracle -> CUDA only)
    osel = torch.from_numpy(np.ascontiguousarray(ref["sel"])).to(run.c.q.device)
    onsel = torch.from_numpy(ref["nsel"]).to(run.c.q.device)
    if osel.shape[2] != run.d.max_sel:
        pad = torch.full((run.d.B, run.d.Hkv, run.d.max_sel), -1, dtype=torch.int32,
                         device=run.c.q.device)
        pad[:, :, :osel.shape[2]] = osel
        osel = pad
    out, lse = run.gpu_decode(osel, onsel)
    errs = {"sparse": assert_out_close(out, lse, ref["out"], ref["lse"], "sparse decode")}
    # again, not right after a selection: both lists in one pass
    out1, lse1 = run.gpu_decode(osel, onsel)
    errs["sparse_one_pass"] = assert_out_close(out1, lse1, ref["out"], ref["lse"],
                                               "sparse decode, one pass")
    assert csa.device_status(run.ws) == 0
    if dense:
        dout, dlse = run.gpu_dense()
        rout, rlse = run.oracle_dense()
        errs["dense"] = assert_out_close(dout, dlse, rout, rlse, "dense decode")
        assert csa.device_status(run.ws) == 0
    return errs


@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K], ids=lambda w: w.name)
def test_workload_parity(w, cuda):
    run = Run(wl.make_case(w, cuda))
    full_check(run)


def test_workload_parity_64k_planted(cuda):
    run = Run(wl.make_case(wl.CTX64K, cuda))
    full_check(run)


# ---------------------------------------------------------------- edge cases
def small(B=2, Hq=8, Hkv=2, D=128, lens=(1000, 777), prefix=20, window=50, budget=160, seed=3,
          extra=0):
    return wl.Workload("edge", B=B, Hq=Hq, Hkv=Hkv, D=D, seq_lens=tuple(lens), prefix=prefix,
                       window=window, budget=budget, seed=seed, steps=extra)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_group_sizes_and_head_dims(G, D, cuda):
    w = small(Hq=2 * G, Hkv=2, D=D, lens=(900, 523))
    full_check(Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("lens,P,W,budget", [
    ((1,), 0, 0, 16),            # one token
    ((15,), 3, 4, 32),           # shorter than a page
    ((16,), 0, 0, 0),            # exactly one page, nothing but prefix/window (empty)
    ((300,), 0, 0, 64),          # no prefix, no window: pure top-k
    ((300,), 17, 33, 0),         # budget 0: prefix + window only, ragged boundaries
    ((300,), 40, 40, 10_000),    # budget covers everything -> dense
    ((300,), 200, 150, 32),      # prefix + window cover everything
    ((257, 1030, 48), 5, 7, 48), # ragged batch, boundary pages partial on both sides
    ((4096 + 5,), 64, 256, 512), # ragged tail page
    ((33,), 17, 15, 16),         # one candidate page partial on both sides
])
def test_edge_geometry(lens, P, W, budget, cuda):
    w = small(B=len(lens), lens=lens, prefix=P, window=W, budget=budget)
    full_check(Run(wl.make_case(w, cuda)))


def test_empty_sequence_outputs_zero(cuda):
    w = small(B=2, lens=(0, 100), prefix=4, window=8, budget=32)
    run = Run(wl.make_case(w, cuda))
    run.gpu_meta()
    run.gpu_select()
    out, lse = run.gpu_decode(run.layer.sel, run.layer.n_sel)
    torch.cuda.synchronize()
    assert (out[0].float() == 0).all() and torch.isneginf(lse[0]).all()
    assert torch.isfinite(out[1].float()).all()
    assert csa.device_status(run.ws) == 0


def test_maximum_budget_and_long_candidate_list(cuda):
    """16k+ candidate pages of one unit, k = 512."""
    w = small(B=1, Hq=8, Hkv=1, D=128, lens=(262144 + 77,), prefix=128, window=512,
              budget=8192)
    run = Run(wl.make_case(w, cuda))
    full_check(run, dense=False)


def test_bad_page_id_sets_device_flag(cuda):
    w = small(B=1, lens=(600,), prefix=16, window=32, budget=64)
    case = wl.make_case(w, cuda)
    run = Run(case)
    run.gpu_meta()
    assert csa.device_status(run.ws) == 0
    case.page_table[0, 5] = w.num_pages + 7        # out of range
    run.gpu_select()
    out, lse = run.gpu_decode(run.layer.sel, run.layer.n_sel)
    flags = csa.device_status(run.ws)
    assert flags & csa.DEVFLAG_BAD_PAGE_ID
    assert csa.device_status(run.ws) == 0           # cleared by the read


def test_bad_selection_sets_device_flag(cuda):
    w = small(B=1, lens=(600,), prefix=16, window=32, budget=64)
    run = Run(wl.make_case(w, cuda))
    run.gpu_meta()
    run.gpu_select()
    sel = run.layer.sel.clone()
    sel[0, 0, 1] = sel[0, 0, 0]                     # not strictly ascending
    run.gpu_decode(sel, run.layer.n_sel)
    assert csa.device_status(run.ws) & csa.DEVFLAG_BAD_SELECTION


# ---------------------------------------------------------------- append
def test_incremental_append_matches_rebuild(cuda):
    """64 single-token appends through csa_meta_update: cache slots hold the
    new tokens and the incremental min/max equals the oracle's recomputation
    on a host cache built by placing the same tokens."""
    steps = 64
    w = small(B=3, Hq=8, Hkv=2, D=128, lens=(1000, 1015, 1024), prefix=16, window=64,
              budget=128, extra=steps)
    case = wl.make_case(w, cuda)
    run = Run(case)
    run.gpu_meta()
    host_k = run.h["k"].copy()
    host_v = run.h["v"].copy()
    pt = run.h["pt"]
    lens = [int(x) for x in run.h["sl"]]
    for step in range(steps):
        q, nk, nv = wl.step_tokens(case, step)
        for b in range(w.B):
            t = lens[b]
            host_k[pt[b, t // PS], :, t % PS] = wl.bits(nk[b, 0])
            host_v[pt[b, t // PS], :, t % PS] = wl.bits(nv[b, 0])
            lens[b] += 1
        case.seq_lens += 1
        csa.meta_update(run.d, case.k_cache, case.v_cache, run.layer.meta, case.page_table,
                        case.seq_lens, nk, nv, 1, run.ws)
    torch.cuda.synchronize()
    assert csa.device_status(run.ws) == 0
    run.h.update(k=host_k, v=host_v, sl=np.array(lens, np.int32))
    # the cache: every appended slot holds the new token
    gk, gv = wl.bits(case.k_cache), wl.bits(case.v_cache)
    for b in range(w.B):
        for t in range(lens[b] - steps, lens[b]):
            phys, slot = pt[b, t // PS], t % PS
            np.testing.assert_array_equal(gk[phys, :, slot], host_k[phys, :, slot])
            np.testing.assert_array_equal(gv[phys, :, slot], host_v[phys, :, slot])
    assert_meta_equal(run, run.layer.meta)


def test_chunk_append_prefill(cuda):
    """A multi-token chunk append (prefill of 333 tokens after 50)."""
    w = small(B=2, Hq=4, Hkv=2, D=64, lens=(50, 50), prefix=8, window=16, budget=64, extra=333)
    case = wl.make_case(w, cuda)
    run = Run(case)
    run.gpu_meta()
    g = torch.Generator(device=cuda).manual_seed(5)
    nk = torch.randn((w.B, 333, w.Hkv, w.D), generator=g, device=cuda).to(torch.bfloat16)
    nv = torch.randn((w.B, 333, w.Hkv, w.D), generator=g, device=cuda).to(torch.bfloat16)
    case.seq_lens += 333
    csa.meta_update(run.d, case.k_cache, case.v_cache, run.layer.meta, case.page_table,
                    case.seq_lens, nk, nv, 333, run.ws)
    torch.cuda.synchronize()
    host_k, pt = run.h["k"].copy(), run.h["pt"]
    nkb = wl.bits(nk)
    for b in range(w.B):
        for i in range(333):
            t = 50 + i
            host_k[pt[b, t // PS], :, t % PS] = nkb[b, i]
    run.h.update(k=host_k, sl=case.seq_lens.cpu().numpy())
    assert_meta_equal(run, run.layer.meta)
    assert csa.device_status(run.ws) == 0


def test_repeat_calls_reuse_workspace(cuda):
    """The same workspace serves many calls: repeated decodes are bit-identical
    (the first, straight after the selection, streams its prefix/window pages
    in a pass of their own and differs by rounding only), and all match the
    oracle."""
    run = Run(wl.make_case(wl.TINY, cuda))
    run.gpu_meta()
    run.gpu_select()
    out1, lse1 = run.gpu_decode(run.layer.sel, run.layer.n_sel)
    outs = [run.gpu_decode(run.layer.sel, run.layer.n_sel) for _ in range(5)]
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])
    ref = run.oracle_step()
    assert_out_close(out1, lse1, ref["out"], ref["lse"], "decode after the selection")
    assert_out_close(outs[0][0], outs[0][1], ref["out"], ref["lse"], "repeated decode")


def test_fixed_pages_streamed_before_the_selection_ends(cuda):
    """Right after csa_score_select on the same stream, the decode streams the
    prefix and window pages while the selection kernel still runs (a pass of
    their own); a decode that waits for everything first takes both lists in
    one pass.  Both match the oracle; repeats of each are bit-identical."""
    run = Run(wl.make_case(wl.CTX32K, cuda))
    run.gpu_meta()
    ref = run.oracle_step()
    osel = torch.from_numpy(np.ascontiguousarray(ref["sel"])).to(cuda)
    onsel = torch.from_numpy(ref["nsel"]).to(cuda)
    prev = None
    for _ in range(3):
        run.gpu_select(scores=False)
        out_e, lse_e = run.gpu_decode(osel, onsel)   # overlapped with the selection
        out_w, lse_w = run.gpu_decode(osel, onsel)   # waits first
        torch.cuda.synchronize()
        assert_out_close(out_e, lse_e, ref["out"], ref["lse"], "early decode")
        assert_out_close(out_w, lse_w, ref["out"], ref["lse"], "waiting decode")
        if prev is not None:
            assert torch.equal(out_e, prev[0]) and torch.equal(out_w, prev[1])
        prev = (out_e, out_w)
    assert csa.device_status(run.ws) == 0


# ---------------------------------------------------------------- one-call path
def sparse_call(run: Run):
    """csa_sparse_attention on the run's layer: (sel, n_sel, out, lse)."""
    d, c = run.d, run.c
    sel = torch.full((d.B, d.Hkv, d.max_sel), -7, dtype=torch.int32, device=c.q.device)
    nsel = torch.full((d.B, d.Hkv), -7, dtype=torch.int32, device=c.q.device)
    out = torch.full((d.B, d.Hq, d.D), float("nan"), dtype=torch.bfloat16, device=c.q.device)
    lse = torch.full((d.B, d.Hq), float("nan"), dtype=torch.float32, device=c.q.device)
    csa.sparse_attention(d, c.q, c.k_cache, c.v_cache, run.layer.meta, c.page_table, c.seq_lens,
                         run.prefix, run.window, run.budget, sel, nsel, out, run.ws, lse)
    return sel, nsel, out, lse


def check_one_call(run: Run, oracle_too=True):
    """The one-call path selects exactly what csa_score_select selects, attends
    like csa_decode on that selection, and matches the oracle: the selection
    by the band rule, and the output of every unit against the oracle's
    attention over that unit's selection (the oracle's own, or, inside a tie
    band, the GPU's valid pick).  Returns the number of units whose selection
    is the oracle's own."""
    run.gpu_meta()
    sel_f, nsel_f, out_f, lse_f = sparse_call(run)
    run.gpu_select(scores=False)
    out_s, lse_s = run.gpu_decode(run.layer.sel, run.layer.n_sel)
    torch.cuda.synchronize()
    assert csa.device_status(run.ws) == 0
    assert torch.equal(nsel_f, run.layer.n_sel)
    for b in range(run.d.B):
        for g in range(run.d.Hkv):
            k = int(nsel_f[b, g])
            assert torch.equal(sel_f[b, g, :k], run.layer.sel[b, g, :k]), f"unit ({b},{g})"
    # the same attention, split differently: bf16 output rounding apart
    err = (out_f.float() - out_s.float()).abs()
    assert torch.isfinite(out_f.float()).all()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
    fin = torch.isfinite(lse_s)
    assert torch.equal(torch.isfinite(lse_f), fin)
    torch.testing.assert_close(lse_f[fin], lse_s[fin], rtol=1e-4, atol=1e-3)
    if not oracle_too:
        return None
    ref = run.oracle_step()
    check_selection(sel_f, nsel_f, ref["scores"], ref["sel"], ref["nsel"])
    exp_out, exp_lse, same = oracle_on_valid_choice(run.od, run.h, run.prefix, run.window,
                                                     run.scale, sel_f, nsel_f, ref)
    assert_out_close(out_f, lse_f, exp_out, exp_lse, "one-call decode")
    G = run.d.Hq // run.d.Hkv
    for b in range(run.d.B):
        for g in range(run.d.Hkv):
            h = slice(g * G, (g + 1) * G)
            assert_out_close(out_f[b, h], lse_f[b, h], exp_out[b, h], exp_lse[b, h],
                             f"one-call decode, unit ({b},{g})")
    return same


@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K, wl.CTX64K], ids=lambda w: w.name)
def test_one_call_parity(w, cuda):
    same = check_one_call(Run(wl.make_case(w, cuda)))
    if w is wl.CTX32K:
        assert same >= 1


@pytest.mark.parametrize("D", [64, 128, 256])
def test_one_call_output_against_oracle(D, cuda):
    """k equal to the number of q-aligned planted pages, one query head per
    kv-head (the plant then stands about 5 sigma above the random pages'
    bounds): the oracle's top-k is unambiguous in most units, and in each of
    them the one-call output is compared with the oracle's attention.  (With 8
    heads per group a plant along the group's summed query stands out much
    less.)"""
    G = 1
    w = wl.Workload("planted_exact", B=3, Hq=2 * G, Hkv=2, D=D, seq_lens=(20000, 13001, 7777),
                    prefix=64, window=512, budget=16 * 12, planted=12, seed=11)
    same = check_one_call(Run(wl.make_case(w, cuda)))
    assert same >= 4


@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_one_call_group_sizes_and_head_dims(G, D, cuda):
    w = small(B=2, Hq=2 * G, Hkv=2, D=D, lens=(3000, 2049), prefix=40, window=100, budget=480)
    check_one_call(Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("lens,P,W,budget", [
    ((1000, 777), 20, 50, 160),        # ragged, partial boundary pages
    ((4096, 16), 0, 0, 256),           # no prefix or window; a one-page sequence
    ((700, 699), 8, 8, 16 * 44),       # budget covers every candidate
    ((513, 2000), 512, 1, 32),         # prefix covers the first sequence
    ((0, 300), 16, 16, 64),            # an empty sequence
    ((333, 4000), 17, 33, 0),          # budget 0: separate kernels
])
def test_one_call_edge_geometry(lens, P, W, budget, cuda):
    w = small(lens=lens, prefix=P, window=W, budget=budget)
    check_one_call(Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_one_call_many_units(G, D, cuda):
    """More than 32 (sequence, kv-head) units: the separate kernels (scoring,
    selection, decode, combine) behind the one call, against the separate
    calls and the oracle, every unit."""
    w = small(B=20, Hq=2 * G, Hkv=2, D=D, lens=tuple(900 + 37 * i for i in range(20)),
              prefix=16, window=64, budget=256)
    check_one_call(Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("lens,P,W,budget", [
    ((0,) * 3 + (700,) * 30, 16, 16, 64),              # empty sequences
    ((40,) * 17 + (1000,) * 16, 16, 32, 64),           # prefix + window cover some sequences
    ((17,) * 11 + (300, 33) * 11, 5, 7, 32),           # candidates fewer than the cluster's CTAs
    ((4096 + 5,) * 33, 64, 256, 512),                  # ragged tail page
    (tuple(600 + 61 * i for i in range(33)), 0, 0, 16),  # no prefix or window, k = 1
])
def test_one_call_many_units_edge_geometry(lens, P, W, budget, cuda):
    w = small(B=len(lens), Hq=4, Hkv=1, lens=lens, prefix=P, window=W, budget=budget)
    check_one_call(Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("B,Hkv", [(8, 4), (16, 2), (11, 3)])
def test_one_call_at_the_fused_unit_limit(B, Hkv, cuda):
    """32 units (the most the single selection + attention launch serves:
    an 8-CTA cluster per unit beside the prefix/window CTAs) and 33 (the
    fewest that take the separate kernels): every unit against the oracle."""
    w = small(B=B, Hq=8 * Hkv, Hkv=Hkv, D=128, lens=tuple(1500 + 97 * i for i in range(B)),
              prefix=16, window=64, budget=256)
    check_one_call(Run(wl.make_case(w, cuda)))


def test_one_call_many_units_ctx64k_batch8(cuda):
    """Batch 8 x 8 kv-heads at 64k (64 units, D = 128), the benchmark's
    larger-batch shape: every unit against the oracle."""
    same = check_one_call(Run(wl.make_case(wl.CTX64K_B8, cuda)))
    assert same >= 32


@pytest.mark.parametrize("window", [0, 15, 16, 64])
def test_one_call_right_after_append(window, cuda):
    """The one-call step issued straight after a one-token append, with the
    appended page inside the window (16 tokens or more) or a candidate
    (fewer): the step equals the same step on metadata rebuilt afterwards,
    bit for bit, and the oracle."""
    w = small(B=2, Hq=8, Hkv=2, D=128, lens=(1000, 1517), prefix=16, window=window,
              budget=128, extra=3)
    case = wl.make_case(w, cuda)
    run = Run(case)
    run.gpu_meta()
    for s in range(3):
        nk, nv = wl.step_tokens(case, s)[1:]
        case.seq_lens += 1
        csa.meta_update(run.d, case.k_cache, case.v_cache, run.layer.meta, case.page_table,
                        case.seq_lens, nk, nv, 1, run.ws)
        sel_a, nsel_a, out_a, lse_a = sparse_call(run)
    torch.cuda.synchronize()
    assert csa.device_status(run.ws) == 0
    meta_after = run.layer.meta.clone()
    run.refresh_host()
    run.gpu_meta()
    assert torch.equal(run.layer.meta, meta_after)
    sel_b, nsel_b, out_b, lse_b = sparse_call(run)
    torch.cuda.synchronize()
    assert torch.equal(nsel_a, nsel_b) and torch.equal(sel_a, sel_b)
    assert torch.equal(out_a, out_b)
    assert torch.equal(torch.isfinite(lse_a), torch.isfinite(lse_b))
    fin = torch.isfinite(lse_b)
    assert torch.equal(lse_a[fin], lse_b[fin])
    check_one_call(run)


def test_one_call_repeated_and_after_appends(cuda):
    """Back-to-back one-call steps with appends in between, no host syncs."""
    w = replace(wl.CTX32K, steps=4)
    case = wl.make_case(w, cuda)
    run = Run(case)
    run.gpu_meta()
    outs = []
    for s in range(4):
        nk, nv = wl.step_tokens(case, s)[1:]
        case.seq_lens += 1
        csa.meta_update(run.d, case.k_cache, case.v_cache, run.layer.meta, case.page_table,
                        case.seq_lens, nk, nv, 1, run.ws)
        outs.append(sparse_call(run))
    torch.cuda.synchronize()
    assert csa.device_status(run.ws) == 0
    run.refresh_host()
    check_one_call(run, oracle_too=False)
