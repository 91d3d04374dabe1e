"""GPU parity at the two largest configurations, checked on samples.

* The 256k stack of the benchmark (batch 4, 32 query / 4 kv heads, D = 128,
  prefix 128): two of its per-layer (window, budget) pairs, 64 decode steps
  that each append one token per sequence (csa_meta_update) and attend
  (csa_sparse_attention).  At a few steps one seeded sequence of each layer is
  copied to the host -- its pages in logical order -- and checked against the
  oracle: metadata bit-exact after the appends, the selection by the band
  rule, and the output of every kv-head against the oracle's attention over
  its selection (the oracle's own, or the GPU's valid pick inside a tie band).
* The ragged sweep (lengths drawn in [4096, 262144]): budgets 0, 1024, 4096
  and "all", every sequence, through the one-call path and the separate calls.
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl
from parity import PS, Run, assert_out_close, check_selection, f64, oracle_on_valid_choice
from test_gpu_parity import check_one_call

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(0)
    yield


def host_sequence(case: wl.Case, meta: torch.Tensor, b: int):
    """Sequence b's pages, in logical order, as a one-sequence host problem:
    (oracle dims, q, k, v, page table, seq_lens, GPU metadata of its pages)."""
    w = case.w
    L = int(case.seq_lens[b])
    np_b = -(-L // PS)
    phys = case.page_table[b, :np_b].long()
    k = wl.bits(case.k_cache[phys])
    v = wl.bits(case.v_cache[phys])
    m = wl.bits(meta[phys])
    q = wl.bits(case.q[b:b + 1])
    d = oracle.Dims(1, w.Hq, w.Hkv, w.D, PS, np_b, np_b)
    pt = np.arange(np_b, dtype=np.int32)[None, :]
    return d, q, k, v, pt, np.array([L], np.int32), m


def check_sequence(case, meta, sel, nsel, out, lse, b, prefix, window, budget, max_sel):
    d, q, k, v, pt, sl, gmeta = host_sequence(case, meta, b)
    ref_meta = oracle.meta(d, k, pt, sl)
    np.testing.assert_array_equal(f64(gmeta), f64(ref_meta), err_msg=f"metadata of sequence {b}")
    ref = oracle.step(d, q, k, v, pt, sl, prefix, window, budget, max_sel,
                      1.0 / math.sqrt(case.w.D))
    gsel = sel[b:b + 1].cpu()
    gn = nsel[b:b + 1].cpu()
    check_selection(gsel, gn, ref["scores"], ref["sel"], ref["nsel"])
    h = dict(q=q, k=k, v=v, pt=pt, sl=sl)
    exp_out, exp_lse, same = oracle_on_valid_choice(d, h, prefix, window,
                                                     1.0 / math.sqrt(case.w.D), gsel, gn, ref)
    G = case.w.Hq // case.w.Hkv
    for g in range(case.w.Hkv):
        hh = slice(g * G, (g + 1) * G)
        assert_out_close(out[b, hh], lse[b, hh], exp_out[0, hh], exp_lse[0, hh],
                         f"sequence {b}, kv-head {g}")
    return same


def test_ctx256k_stack_with_appends_sampled(cuda):
    steps, check_at = 64, (0, 31, 63)
    w = replace(wl.CTX256K, steps=steps)
    rng = np.random.default_rng(1234)
    compared = 0
    for layer in (0, 3):                        # (512, 1024) and (4096, 8192)
        case = wl.make_case(w, cuda, layer=layer)
        d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
        lay = csa.Layer(d, case.k_cache, case.v_cache, case.page_table, case.seq_lens,
                        w.prefix, case.window, case.budget)
        lay.rebuild_meta()
        for s in range(steps):
            q, nk, nv = wl.step_tokens(case, s)
            case.seq_lens += 1
            case.q = q
            out = lay.step(q, nk, nv, fused=True)
            if s in check_at:
                torch.cuda.synchronize()
                assert csa.device_status(lay.ws) == 0
                b = int(rng.integers(w.B))
                compared += check_sequence(case, lay.meta, lay.sel, lay.n_sel, out, lay.lse, b,
                                           w.prefix, case.window, case.budget, d.max_sel)
        del case, lay
        torch.cuda.empty_cache()
    assert compared >= 6          # most sampled units have an unambiguous selection


@pytest.mark.parametrize("budget", [0, 1024, 4096, None], ids=["b0", "b1024", "b4096", "all"])
def test_ragged_sweep(budget, cuda):
    w = wl.SWEEP
    if budget is None:
        budget = PS * w.max_pages                # every candidate page ("all")
    case = wl.make_case(w, cuda)
    run = Run(case, budget=budget)
    same = check_one_call(run)
    if budget in (0, PS * w.max_pages):
        assert same == w.B * w.Hkv               # the selection is forced
