"""GPU parity of the context-parallel step, with the ranks emulated in one
process on one GPU: every rank's calls run in turn on its shard of one cache
(the shard's page-table columns), and the all-gathers are lists.  Checked:
the merge kernel against the log-sum-exp merge written out in numpy, the
shard kernel against a filter, csa_select_scores against csa_score_select's
own selection, and the whole step against the one-GPU call and the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import context_parallel as cp
from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl
from parity import PS, Run, assert_out_close, check_selection, oracle_on_valid_choice
from test_context_parallel import ListExchange, lse_merge

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(0)
    yield


@pytest.mark.parametrize("R,D", [(1, 64), (2, 128), (3, 256), (8, 128)])
def test_merge_kernel(R, D, cuda):
    g = torch.Generator(device="cpu").manual_seed(R * 1000 + D)
    B, Hq = 3, 5
    outs = torch.randn((R, B, Hq, D), generator=g).to(torch.bfloat16)
    lses = torch.randn((R, B, Hq), generator=g) * 3
    if R > 1:
        lses[0, 0, 1] = float("-inf")            # a part that attended nothing
    lses[:, 1, 2] = float("-inf")                # a head nobody attended
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=cuda)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=cuda)
    csa.merge_attention(outs.to(cuda), lses.to(cuda), out, lse)
    torch.cuda.synchronize()
    ref_out, ref_lse = lse_merge(list(outs.double().numpy()), list(lses.double().numpy()))
    got = out.cpu().double().numpy()
    # fp32 arithmetic, one bf16 rounding of the result
    np.testing.assert_allclose(got, ref_out, rtol=2 ** -8, atol=1e-6)
    fin = np.isfinite(ref_lse)
    np.testing.assert_array_equal(np.isfinite(lse.cpu().numpy()), fin)
    np.testing.assert_allclose(lse.cpu().numpy()[fin], ref_lse[fin], rtol=1e-6, atol=1e-5)
    assert not got[1, 2].any()


def test_shard_selection_kernel(cuda):
    rng = np.random.default_rng(5)
    B, Hkv, max_sel = 3, 2, 40
    d = csa.make_dims(B, 4, Hkv, 64, 300, 1000, max_sel)
    sel = np.full((B, Hkv, max_sel), -1, np.int32)
    n = rng.integers(0, max_sel + 1, size=(B, Hkv)).astype(np.int32)
    for b in range(B):
        for h in range(Hkv):
            sel[b, h, :n[b, h]] = np.sort(rng.choice(300, size=n[b, h], replace=False))
    for lo, hi in ((0, 100), (100, 220), (220, 300), (50, 50)):
        sl = torch.full((B, Hkv, max_sel + 3), -7, dtype=torch.int32, device=cuda)
        nl = torch.full((B, Hkv), -7, dtype=torch.int32, device=cuda)
        csa.shard_selection(d, torch.from_numpy(sel).to(cuda), torch.from_numpy(n).to(cuda), lo,
                            hi, sl, nl)
        torch.cuda.synchronize()
        gs, gn = sl.cpu().numpy(), nl.cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                p = sel[b, h, :n[b, h]]
                p = p[(p >= lo) & (p < hi)] - lo
                assert gn[b, h] == len(p)
                np.testing.assert_array_equal(gs[b, h, :len(p)], p)


@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K], ids=lambda w: w.name)
def test_select_scores_equals_score_select(w, cuda):
    run = Run(wl.make_case(w, cuda))
    run.gpu_meta()
    sc = torch.full((run.d.B, run.d.Hkv, run.d.max_pages_per_seq), float("nan"), device=cuda)
    lay = run.layer
    csa.score_select(run.d, run.c.q, lay.meta, run.c.page_table, run.c.seq_lens, run.prefix,
                     run.window, run.budget, lay.sel, lay.n_sel, run.ws, scores_out=sc)
    sel2 = torch.full_like(lay.sel, -5)
    n2 = torch.full_like(lay.n_sel, -5)
    csa.select_scores(run.d, sc, run.c.seq_lens, run.prefix, run.window, run.budget, sel2, n2,
                      run.ws)
    torch.cuda.synchronize()
    assert csa.device_status(run.ws) == 0
    assert torch.equal(n2, lay.n_sel)
    for b in range(run.d.B):
        for h in range(run.d.Hkv):
            k = int(n2[b, h])
            assert torch.equal(sel2[b, h, :k], lay.sel[b, h, :k])


@pytest.mark.parametrize("noalloc", [False, True], ids=["decode", "decode_noalloc"])
def test_decode_straight_after_select_scores(noalloc, cuda):
    """csa_decode (and csa_decode_noalloc) issued straight after
    csa_select_scores on the same stream, no host sync in between: the
    selection kernel lets the next grid start before it writes the selection,
    so the decode must read it only after its dependency wait.  Repeated, the
    outputs match the oracle's attention over the (band-valid) selection."""
    run = Run(wl.make_case(wl.CTX32K, cuda))
    run.gpu_meta()
    sc = torch.full((run.d.B, run.d.Hkv, run.d.max_pages_per_seq), float("nan"), device=cuda)
    lay = run.layer
    csa.score_select(run.d, run.c.q, lay.meta, run.c.page_table, run.c.seq_lens, run.prefix,
                     run.window, run.budget, lay.sel, lay.n_sel, run.ws, scores_out=sc)
    ref = run.oracle_step()
    for _ in range(3):
        sel2 = torch.full_like(lay.sel, -5)
        n2 = torch.full_like(lay.n_sel, -5)
        out = torch.empty((run.d.B, run.d.Hq, run.d.D), dtype=torch.bfloat16, device=cuda)
        lse = torch.empty((run.d.B, run.d.Hq), dtype=torch.float32, device=cuda)
        csa.select_scores(run.d, sc, run.c.seq_lens, run.prefix, run.window, run.budget, sel2,
                          n2, run.ws)
        if noalloc:
            csa.decode_noalloc(run.d, run.c.q, run.c.k_cache, run.c.v_cache, run.c.page_table,
                               run.c.seq_lens, sel2, n2, run.prefix, run.window, out, lse)
        else:
            csa.decode(run.d, run.c.q, run.c.k_cache, run.c.v_cache, run.c.page_table,
                       run.c.seq_lens, sel2, n2, run.prefix, run.window, out, run.ws, lse)
        torch.cuda.synchronize()
        assert csa.device_status(run.ws) == 0
        check_selection(sel2, n2, ref["scores"], ref["sel"], ref["nsel"])
        exp_out, exp_lse, _ = oracle_on_valid_choice(run.od, run.h, run.prefix, run.window,
                                                     run.scale, sel2, n2, ref)
        assert_out_close(out, lse, exp_out, exp_lse, "decode after csa_select_scores")


def emulate(run: Run, R: int):
    """The R ranks' steps on one GPU; returns (out, lse, sel, n_sel)."""
    c, w = run.c, run.c.w
    sl_host = c.seq_lens.cpu().tolist()
    plan = cp.plan_shards(w.max_pages, R, run.prefix, run.window, sl_host)
    meta = run.layer.meta
    ops = [cp.CudaOps(plan, run.d, cp.shard_from_global(plan, r, c.k_cache, c.v_cache, meta,
                                                         c.page_table, sl_host),
                      c.seq_lens, run.prefix, run.window, run.budget, run.scale)
           for r in range(R)]
    scores = [o.local_scores(c.q).clone() for o in ops]
    parts = []
    for o in ops:
        s = cp.gather_scores(ListExchange(scores_padded(scores, plan)), plan, scores[o.sh.rank])
        out_r, lse_r = o.attend(c.q, s)
        parts.append((out_r.clone(), lse_r.clone()))
    out, lse = ops[0].merge([p[0] for p in parts], [p[1] for p in parts])
    torch.cuda.synchronize()
    for o in ops:
        assert csa.device_status(o.ws_local) == 0
        assert csa.device_status(o.ws_global) == 0
        assert torch.equal(o.sel, ops[0].sel) and torch.equal(o.n_sel, ops[0].n_sel)
    return out, lse, ops[0].sel, ops[0].n_sel


def scores_padded(scores, plan):
    width = max(plan.hi(r) - plan.lo(r) for r in range(plan.world))
    out = []
    for s in scores:
        if s.shape[2] < width:
            s = torch.cat([s, s.new_full(s.shape[:2] + (width - s.shape[2],), float("nan"))], 2)
        out.append(s)
    return out


@pytest.mark.parametrize("R", [2, 3])
@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K], ids=lambda w: w.name)
def test_context_parallel_step(w, R, cuda):
    run = Run(wl.make_case(w, cuda))
    run.gpu_meta()
    out, lse, sel, n_sel = emulate(run, R)
    # the one-GPU call on the same cache
    lay = run.layer
    out1 = torch.empty_like(out)
    lse1 = torch.empty_like(lse)
    csa.sparse_attention(run.d, run.c.q, run.c.k_cache, run.c.v_cache, lay.meta,
                         run.c.page_table, run.c.seq_lens, run.prefix, run.window, run.budget,
                         lay.sel, lay.n_sel, out1, run.ws, lse=lse1, scale=run.scale)
    torch.cuda.synchronize()
    assert torch.equal(n_sel, lay.n_sel)
    for b in range(run.d.B):
        for h in range(run.d.Hkv):
            k = int(n_sel[b, h])
            assert torch.equal(sel[b, h, :k], lay.sel[b, h, :k]), f"unit ({b},{h})"
    err = (out.float() - out1.float()).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
    torch.testing.assert_close(lse, lse1, rtol=1e-4, atol=1e-3)
    # and against the oracle, in every unit whose selection is the oracle's
    ref = run.oracle_step()
    check_selection(sel, n_sel, ref["scores"], ref["sel"], ref["nsel"])
    gs, gn = sel.cpu().numpy(), n_sel.cpu().numpy()
    G = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hkv):
            k = int(gn[b, h])
            if np.array_equal(gs[b, h, :k], ref["sel"][b, h, :k]):
                hh = slice(h * G, (h + 1) * G)
                assert_out_close(out[b, hh], lse[b, hh], ref["out"][b, hh], ref["lse"][b, hh],
                                 f"context-parallel, unit ({b},{h})")
