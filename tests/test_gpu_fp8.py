"""GPU parity of the optional fp8 metadata path against the oracle's fp8
definition (csa_oracle.c): the fp8 copy bit-exact (after a rebuild and after
appends), scores to fp32 accuracy, the selection by the band rule, and the
one-call output of every unit against the oracle's attention over that unit's
selection (the oracle's own, or the GPU's valid pick inside a tie band)."""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl
from parity import (PS, assert_out_close, assert_scores_close, check_selection,
                    oracle_on_valid_choice)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(0)
    yield


class Fp8Run:
    def __init__(self, case: wl.Case, budget=None):
        self.c = c = case
        w = case.w
        self.budget = case.budget if budget is None else budget
        self.max_sel = max(1, max(w.max_sel, self.budget // PS))
        self.d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, self.max_sel)
        self.od = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
        self.layer = csa.Layer(self.d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix,
                               case.window, self.budget, fp8=True)
        self.layer.rebuild_meta()

    def host(self):
        c = self.c
        return dict(q=wl.bits(c.q), k=wl.bits(c.k_cache), v=wl.bits(c.v_cache),
                    pt=c.page_table.cpu().numpy(), sl=c.seq_lens.cpu().numpy())

    def oracle_meta8(self, h):
        m = oracle.meta(self.od, h["k"], h["pt"], h["sl"])
        return oracle.meta_fp8(self.od, m, h["pt"], h["sl"])


def assert_meta8_equal(run: Fp8Run, h):
    ref = run.oracle_meta8(h)
    got = run.layer.meta8.cpu().numpy()
    for b in range(run.d.B):
        np_b = -(-int(h["sl"][b]) // PS)
        phys = h["pt"][b, :np_b]
        np.testing.assert_array_equal(got[phys], ref[phys], err_msg=f"fp8 metadata, sequence {b}")


def check_fp8(run: Fp8Run, one_call=True):
    h = run.host()
    assert_meta8_equal(run, h)
    w = run.c.w
    ref = oracle.step_fp8(run.od, h["q"], h["k"], h["v"], h["pt"], h["sl"], w.prefix,
                          run.c.window, run.budget, run.max_sel, 1.0 / math.sqrt(w.D))
    sc = torch.full((run.d.B, run.d.Hkv, run.d.max_pages_per_seq), float("nan"),
                    dtype=torch.float32, device=run.c.q.device)
    lay = run.layer
    csa.score_select_fp8(run.d, run.c.q, lay.meta8, run.c.page_table, run.c.seq_lens, w.prefix,
                         run.c.window, run.budget, lay.sel, lay.n_sel, lay.ws, scores_out=sc)
    torch.cuda.synchronize()
    assert_scores_close(sc, ref["scores"])
    check_selection(lay.sel, lay.n_sel, ref["scores"], ref["sel"], ref["nsel"], gpu_scores=sc)
    sel_s, nsel_s = lay.sel.clone(), lay.n_sel.clone()
    if not one_call:
        return 0
    out = lay.step(run.c.q, fused=True)
    torch.cuda.synchronize()
    assert csa.device_status(lay.ws) == 0
    assert torch.equal(lay.n_sel, nsel_s)
    gs, gn = lay.sel.cpu().numpy(), lay.n_sel.cpu().numpy()
    assert all(np.array_equal(gs[b, g, :gn[b, g]], sel_s.cpu().numpy()[b, g, :gn[b, g]])
               for b in range(run.d.B) for g in range(run.d.Hkv))
    exp_out, exp_lse, same = oracle_on_valid_choice(run.od, h, w.prefix, run.c.window,
                                                     1.0 / math.sqrt(w.D), lay.sel, lay.n_sel,
                                                     ref)
    G = w.Hq // w.Hkv
    for b in range(run.d.B):
        for g in range(run.d.Hkv):
            hh = slice(g * G, (g + 1) * G)
            assert_out_close(out[b, hh], lay.lse[b, hh], exp_out[b, hh], exp_lse[b, hh],
                             f"fp8 one-call, unit ({b},{g})")
    return same


@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K, wl.CTX64K], ids=lambda w: w.name)
def test_fp8_parity(w, cuda):
    same = check_fp8(Fp8Run(wl.make_case(w, cuda)))
    if w is not wl.TINY:
        assert same >= 1


@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_fp8_group_sizes_and_head_dims(G, D, cuda):
    w = wl.Workload("fp8", B=2, Hq=2 * G, Hkv=2, D=D, seq_lens=(3000, 2049), prefix=40,
                    window=100, budget=480, seed=13)
    check_fp8(Fp8Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("Hkv,D,G", [(4, 64, 1), (4, 128, 8), (4, 128, 16), (4, 256, 2),
                                     (4, 256, 16), (8, 64, 8), (8, 128, 1), (8, 128, 16)])
def test_fp8_page_major_shapes(Hkv, D, G, cuda):
    """Shapes whose fp8 scores come from the page-major kernel (4 or 8
    kv-heads; 4 at D = 256): many ragged sequences, some without candidates,
    so that CTA ranges start, end and change sequence inside 16-page groups."""
    lens = (3000, 2049, 17, 800, 4096, 1, 1500, 2200)
    w = wl.Workload("fp8_pm", B=len(lens), Hq=Hkv * G, Hkv=Hkv, D=D, seq_lens=lens, prefix=40,
                    window=100, budget=480, seed=19)
    check_fp8(Fp8Run(wl.make_case(w, cuda)))


@pytest.mark.parametrize("Hkv", [2, 4])
def test_fp8_scores_with_subnormal_rows(Hkv, cuda):
    """Keys whose channel 0 is about 256 and whose other channels lie within
    2^-8: every fp8 row keeps exponent 0, so the small channels are E4M3
    subnormals (below 2^-6).  Their share of a score is about 2^-9 of it,
    far above the tolerance, so the scores match the oracle's fp8 definition
    only if no stage of the kernel drops a subnormal (4 kv-heads: the
    page-major kernel; 2: the ring)."""
    w = wl.Workload("fp8_subnormal", B=2, Hq=4 * Hkv, Hkv=Hkv, D=128, seq_lens=(3000, 2049),
                    prefix=40, window=100, budget=480, seed=23)
    case = wl.make_case(w, cuda)
    g = torch.Generator(device=cuda).manual_seed(29)
    k = (torch.rand(case.k_cache.shape, generator=g, device=cuda) * 2 - 1) * 2.0 ** -8
    sign = torch.randint(0, 2, case.k_cache.shape[:-1], generator=g, device=cuda) * 2 - 1
    k[..., 0] = 256.0 * sign
    case.k_cache.copy_(k.to(torch.bfloat16))
    run = Fp8Run(case)
    h = run.host()
    assert_meta8_equal(run, h)
    m8 = run.oracle_meta8(h)
    # the small channels are E4M3 subnormals: exponent field 0, mantissa nonzero
    used = np.concatenate([h["pt"][b, :-(-int(h["sl"][b]) // PS)] for b in range(w.B)])
    body = m8[used][:, :, np.r_[1:w.D, w.D + 1:2 * w.D]]
    assert ((body & 0x78) == 0).mean() > 0.9 and ((body & 0x07) != 0).mean() > 0.5
    ref = oracle.scores_fp8(run.od, h["q"], m8, h["pt"], h["sl"], w.prefix, case.window)
    lay = run.layer
    sc = torch.full((run.d.B, run.d.Hkv, run.d.max_pages_per_seq), float("nan"),
                    dtype=torch.float32, device=cuda)
    csa.score_select_fp8(run.d, case.q, lay.meta8, case.page_table, case.seq_lens, w.prefix,
                         case.window, run.budget, lay.sel, lay.n_sel, lay.ws, scores_out=sc)
    torch.cuda.synchronize()
    assert csa.device_status(lay.ws) == 0
    assert_scores_close(sc, ref)


def test_fp8_copy_after_appends_matches_rebuild(cuda):
    """64 single-token appends through csa_meta_update_fp8: the fp8 copy is
    the oracle's from the final cache, bit for bit."""
    w = replace(wl.CTX32K, steps=64)
    case = wl.make_case(w, cuda)
    run = Fp8Run(case)
    d, lay = run.d, run.layer
    for s in range(64):
        _, nk, nv = wl.step_tokens(case, s)
        case.seq_lens += 1
        csa.meta_update_fp8(d, case.k_cache, case.v_cache, lay.meta, lay.meta8, case.page_table,
                            case.seq_lens, nk, nv, 1, lay.ws)
    torch.cuda.synchronize()
    assert csa.device_status(lay.ws) == 0
    assert_meta8_equal(run, run.host())


def test_fp8_scores_bound_the_bf16_scores(cuda):
    """On the GPU, too: the fp8 score of every candidate is at least its bf16
    score (the box only grows)."""
    case = wl.make_case(wl.CTX32K, cuda)
    run = Fp8Run(case)
    d, lay, w = run.d, run.layer, case.w
    s8 = torch.full((d.B, d.Hkv, d.max_pages_per_seq), float("nan"), device=cuda)
    s16 = torch.full_like(s8, float("nan"))
    csa.score_select_fp8(d, case.q, lay.meta8, case.page_table, case.seq_lens, w.prefix,
                         case.window, run.budget, lay.sel, lay.n_sel, lay.ws, scores_out=s8)
    csa.score_select(d, case.q, lay.meta, case.page_table, case.seq_lens, w.prefix, case.window,
                     run.budget, lay.sel, lay.n_sel, lay.ws, scores_out=s16)
    torch.cuda.synchronize()
    cand = ~torch.isnan(s16)
    assert torch.equal(cand, ~torch.isnan(s8))
    # fp32 sums of exact products: allow their rounding
    assert (s8[cand] >= s16[cand] - 1e-5 * s16[cand].abs() - 1e-3).all()


def test_fp8_scores_for_extreme_query_magnitudes(cuda):
    """Query components far below 2^-17 and far above the f16 range (65504),
    per head and mixed within one head: the scores from the fp8 copy still
    match the oracle's fp8 definition (exact bf16 q, fp64), relative to each
    unit's own magnitude, and the selection follows the band rule."""
    w = wl.Workload("fp8_qrange", B=2, Hq=16, Hkv=4, D=128, seq_lens=(3000, 2049), prefix=40,
                    window=100, budget=480, seed=17)
    case = wl.make_case(w, cuda)
    G = w.G
    chan = torch.arange(w.D, device=cuda, dtype=torch.float32)
    q = case.q.float()
    q[:, 0 * G:1 * G] *= 2.0 ** -30                          # every component tiny
    q[:, 1 * G:2 * G] *= 2.0 ** 24                           # beyond f16's largest value
    q[:, 2 * G:3 * G] *= torch.exp2(chan % 64 - 44.0)        # 2^-44 .. 2^19 within each head
    case.q = q.to(torch.bfloat16)                            # kv-head 3 as drawn
    run = Fp8Run(case)
    h = run.host()
    assert_meta8_equal(run, h)
    m8 = run.oracle_meta8(h)
    ref = oracle.scores_fp8(run.od, h["q"], m8, h["pt"], h["sl"], w.prefix, case.window)
    lay = run.layer
    sc = torch.full((run.d.B, run.d.Hkv, run.d.max_pages_per_seq), float("nan"),
                    dtype=torch.float32, device=cuda)
    csa.score_select_fp8(run.d, case.q, lay.meta8, case.page_table, case.seq_lens, w.prefix,
                         case.window, run.budget, lay.sel, lay.n_sel, lay.ws, scores_out=sc)
    torch.cuda.synchronize()
    assert csa.device_status(lay.ws) == 0
    got = sc.cpu().numpy().astype(np.float64)
    cand = ~np.isnan(ref)
    assert np.array_equal(~np.isnan(got), cand)
    for b in range(w.B):
        for g in range(w.Hkv):
            c = cand[b, g]
            r, x = ref[b, g][c], got[b, g][c]
            scale = np.abs(r).max()
            assert scale > 0 and np.isfinite(x).all(), f"unit ({b},{g})"
            np.testing.assert_allclose(x, r, rtol=2e-5, atol=1e-6 * scale,
                                       err_msg=f"fp8 scores, unit ({b},{g})")
    sel, nsel = oracle.select(run.od, ref, h["sl"], w.prefix, case.window, run.budget,
                              run.max_sel)
    check_selection(lay.sel, lay.n_sel, ref, sel, nsel, gpu_scores=sc)
