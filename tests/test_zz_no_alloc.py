"""csa_decode_noalloc, the decode entry point for callers that cannot
allocate device memory (a plugin inside a runtime that owns every device
buffer, or a server that reserves the whole GPU at start-up): its scratch
is a fixed array inside the library instead of a caller workspace.

Called through the C ABI twice in a row, it must give what csa_decode gives
on the same inputs, and the oracle's attention, within the attention
tolerance of the parity tests; a small call straight after a large one must
not read what the large one left in the shared scratch; a shape whose
scratch exceeds the array is refused before anything is launched.  This
file is collected last so that a failure here never hides the others; it
passes alone in a fresh process and after the rest of the suite."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl
from parity import PS, assert_out_close

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3      # the parity tests' attention tolerance


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(0)
    yield


def close(a, b):
    err = (a.float() - b.float()).abs()
    return err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


def oracle_problem(c, w):
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
    h = dict(q=wl.bits(c.q), k=wl.bits(c.k_cache), v=wl.bits(c.v_cache),
             pt=c.page_table.cpu().numpy(), sl=c.seq_lens.cpu().numpy())
    ref = oracle.step(od, h["q"], h["k"], h["v"], h["pt"], h["sl"], w.prefix, w.window,
                      w.budget, max(1, w.max_sel), 1.0 / math.sqrt(w.D))
    return od, h, ref


def oracle_selection(ref, d, dev):
    """The oracle's page selection as device tensors of the call's width."""
    sel = torch.full((d.B, d.Hkv, d.max_sel), -1, dtype=torch.int32, device=dev)
    osel = torch.from_numpy(np.ascontiguousarray(ref["sel"]))
    sel[:, :, :osel.shape[2]] = osel.to(dev)
    return sel, torch.from_numpy(ref["nsel"]).to(dev)


def noalloc(d, c, w, sel, nsel):
    out = torch.full((d.B, d.Hq, d.D), float("nan"), dtype=torch.bfloat16, device=c.q.device)
    lse = torch.full((d.B, d.Hq), float("nan"), dtype=torch.float32, device=c.q.device)
    csa.decode_noalloc(d, c.q, c.k_cache, c.v_cache, c.page_table, c.seq_lens, sel, nsel,
                       w.prefix, w.window, out, lse)
    return out, lse


@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K], ids=lambda w: w.name)
def test_noalloc_decode_matches_workspace_decode_and_oracle(w):
    dev = torch.device("cuda:0")
    c = wl.make_case(w, dev)
    d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
    od, h, ref = oracle_problem(c, w)
    sel, nsel = oracle_selection(ref, d, dev)
    # the workspace decode on the same (oracle) selection
    ws = csa.new_workspace(d, dev)
    want = torch.empty((d.B, d.Hq, d.D), dtype=torch.bfloat16, device=dev)
    want_lse = torch.empty((d.B, d.Hq), dtype=torch.float32, device=dev)
    csa.decode(d, c.q, c.k_cache, c.v_cache, c.page_table, c.seq_lens, sel, nsel, w.prefix,
               w.window, want, ws, want_lse)
    for _ in range(2):
        out, lse = noalloc(d, c, w, sel, nsel)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert close(out, want)
        torch.testing.assert_close(lse, want_lse, rtol=1e-4, atol=1e-3)
        assert_out_close(out, lse, ref["out"], ref["lse"], f"csa_decode_noalloc, {w.name}")
    assert csa.device_status(ws) == 0


def test_noalloc_small_call_after_large_call():
    """A call with fewer units, an empty sequence and a unit that selected
    nothing, straight after a 32k call that filled the scratch with its own
    record ranges and partial results: the small call reads none of them."""
    dev = torch.device("cuda:0")
    big = wl.CTX32K
    cb = wl.make_case(big, dev)
    db = csa.make_dims(big.B, big.Hq, big.Hkv, big.D, big.max_pages, big.num_pages, big.max_sel)
    _, _, refb = oracle_problem(cb, big)
    selb, nselb = oracle_selection(refb, db, dev)
    small = wl.Workload("small_after_large", B=3, Hq=4, Hkv=1, D=128, seq_lens=(0, 700, 40),
                        prefix=16, window=32, budget=64, seed=21)
    cs = wl.make_case(small, dev)
    ds = csa.make_dims(small.B, small.Hq, small.Hkv, small.D, small.max_pages, small.num_pages,
                       small.max_sel)
    od, h, refs = oracle_problem(cs, small)
    assert int(refs["nsel"][2, 0]) == 0            # prefix + window cover sequence 2
    sels, nsels = oracle_selection(refs, ds, dev)
    for _ in range(2):
        outb, lseb = noalloc(db, cb, big, selb, nselb)
        outs, lses = noalloc(ds, cs, small, sels, nsels)
        torch.cuda.synchronize()
        assert_out_close(outb, lseb, refb["out"], refb["lse"], "large call")
        assert (outs[0].float() == 0).all() and torch.isneginf(lses[0]).all()
        assert_out_close(outs[1:], lses[1:], refs["out"][1:], refs["lse"][1:],
                         "small call after the large one")


def test_noalloc_refuses_shapes_beyond_its_scratch():
    """Sequences x kv-heads beyond what the built-in scratch holds (about 560
    at D = 128, 8 query heads per kv-head, on 148 SMs): CSA_ERR_WORKSPACE,
    with nothing launched (the output keeps its contents); the largest batch
    that fits still decodes correctly."""
    dev = torch.device("cuda:0")
    Hkv, G, D, L = 8, 8, 128, 40

    def call(B):
        w = wl.Workload("noalloc_limit", B=B, Hq=G * Hkv, Hkv=Hkv, D=D, seq_lens=(L,) * B,
                        prefix=8, window=8, budget=16, seed=5)
        c = wl.make_case(w, dev)
        d = csa.make_dims(B, w.Hq, Hkv, D, w.max_pages, w.num_pages, w.max_sel)
        sel = torch.zeros((B, Hkv, d.max_sel), dtype=torch.int32, device=dev)
        nsel = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)   # prefix + window only
        out = torch.full((B, w.Hq, D), 7.0, dtype=torch.bfloat16, device=dev)
        try:
            csa.decode_noalloc(d, c.q, c.k_cache, c.v_cache, c.page_table, c.seq_lens, sel,
                               nsel, w.prefix, w.window, out)
        except csa.CsaError as e:
            torch.cuda.synchronize()
            assert e.status == csa.CSA_ERR_WORKSPACE
            assert (out.float() == 7.0).all()
            return None
        torch.cuda.synchronize()
        return w, c, sel, nsel, out

    assert call(200) is None                       # 1600 units: refused
    lo, hi = 1, 200                                # call(lo) fits, call(hi) does not
    assert call(lo) is not None
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if call(mid) is None:
            hi = mid
        else:
            lo = mid
    assert lo * Hkv >= 400                         # a few hundred units fit
    w, c, sel, nsel, out = call(lo)
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
    h = dict(q=wl.bits(c.q), k=wl.bits(c.k_cache), v=wl.bits(c.v_cache),
             pt=c.page_table.cpu().numpy(), sl=c.seq_lens.cpu().numpy())
    ref_out, _ = oracle.attend(od, h["q"], h["k"], h["v"], h["pt"], h["sl"], w.prefix, w.window,
                               None, None, 1, 1.0 / math.sqrt(D))
    err = np.abs(out.float().cpu().numpy() - ref_out.astype(np.float32))
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
