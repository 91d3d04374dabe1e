"""The hand-derived worked example in tests/golden/quest_tie_example.json:
the oracle (CPU) and the CUDA path (GPU) against values that follow from the
method's definitions by hand (the Quest page bound with the max over the GQA
group, ties to the lower page, softmax over prefix, window and the selected
page).  The example has two live channels; the other channels are zero, so
the same case runs at the CUDA path's head dims."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
D = 64                       # two live channels, the rest zero


def load():
    with open(os.path.join(HERE, "golden", "quest_tie_example.json")) as f:
        return json.load(f)


def bf16_bits(x):
    """float32 values exactly representable in bf16 -> uint16 bits."""
    a = np.asarray(x, np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def build(ex):
    """Host arrays of the example: q [1][2][D], k/v [5][1][16][D], page
    table [1][5], seq_lens [1] (bf16 as uint16 bits)."""
    ps, pt = ex["page_size"], np.array([ex["page_table"]], np.int32)
    n_pages = pt.shape[1]
    q = np.zeros((1, 2, D), np.float32)
    q[0, :, :2] = ex["q"]
    k = np.zeros((n_pages, 1, ps, D), np.float32)
    v = np.zeros((n_pages, 1, ps, D), np.float32)
    for page in range(n_pages):
        phys = pt[0, page]
        for t in range(ps):
            k[phys, 0, t, :2] = ex["keys_even"][page] if t % 2 == 0 else ex["keys_odd"][page]
            v[phys, 0, t, :2] = ex["values"][page]
    for a in (q, k, v):                            # every value is exact in bf16
        assert (bf16_bits(a).astype(np.uint32) << 16).view(np.float32).tolist() == a.tolist()
    sl = np.array([ex["seq_len"]], np.int32)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v), pt, sl


def test_fixture_is_consistent():
    """The stored numbers are the closed forms the fixture states."""
    ex = load()
    c1, c2 = np.cosh(1.0), np.cosh(2.0)
    np.testing.assert_allclose(ex["expected_out"], [[0, c1 / (2 + c1)], [0, c2 / (2 + c2)]],
                               rtol=1e-15)
    np.testing.assert_allclose(ex["expected_lse"], [np.log(32 + 16 * c1), np.log(32 + 16 * c2)],
                               rtol=1e-15)


def test_oracle_on_the_worked_example():
    ex = load()
    q, k, v, pt, sl = build(ex)
    d = oracle.Dims(1, 2, 1, D, ex["page_size"], pt.shape[1], pt.shape[1])
    P, W, budget = ex["prefix"], ex["window"], ex["budget"]
    sc = oracle.scores(d, q, k, pt, sl, P, W)
    for page, want in ex["expected_scores"].items():
        assert sc[0, 0, int(page)] == want
    assert np.isnan(sc[0, 0, 0]) and np.isnan(sc[0, 0, 4])      # prefix and window pages
    sel, nsel = oracle.select(d, sc, sl, P, W, budget, 4)
    assert nsel[0, 0] == len(ex["expected_selection"])
    assert sel[0, 0, :nsel[0, 0]].tolist() == ex["expected_selection"]
    out, lse = oracle.attend(d, q, k, v, pt, sl, P, W, sel, nsel, 4, 1.0)
    np.testing.assert_allclose(out[0, :, :2], ex["expected_out"], rtol=1e-13, atol=1e-15)
    assert not out[0, :, 2:].any()
    np.testing.assert_allclose(lse[0], ex["expected_lse"], rtol=1e-13)


@pytest.mark.gpu
@pytest.mark.parametrize("one_call", [True, False])
def test_cuda_path_on_the_worked_example(one_call):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_b200 import csa
    ex = load()
    q, k, v, pt, sl = build(ex)
    dev = torch.device("cuda:0")
    t = lambda a, dt: torch.from_numpy(a.astype(dt)).to(dev)
    qd = t(q, np.int16).view(torch.bfloat16)
    kd = t(k, np.int16).view(torch.bfloat16)
    vd = t(v, np.int16).view(torch.bfloat16)
    ptd, sld = t(pt, np.int32), t(sl, np.int32)
    n_pages = pt.shape[1]
    d = csa.make_dims(1, 2, 1, D, n_pages, n_pages, 4)
    lay = csa.Layer(d, kd, vd, ptd, sld, ex["prefix"], ex["window"], ex["budget"])
    lay.rebuild_meta()
    sel = torch.full((1, 1, 4), -7, dtype=torch.int32, device=dev)
    nsel = torch.full((1, 1), -7, dtype=torch.int32, device=dev)
    out = torch.empty((1, 2, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 2), dtype=torch.float32, device=dev)
    if one_call:
        csa.sparse_attention(d, qd, kd, vd, lay.meta, ptd, sld, ex["prefix"], ex["window"],
                             ex["budget"], sel, nsel, out, lay.ws, lse, scale=1.0)
    else:
        scores = torch.full((1, 1, n_pages), float("nan"), device=dev)
        csa.score_select(d, qd, lay.meta, ptd, sld, ex["prefix"], ex["window"], ex["budget"],
                         sel, nsel, lay.ws, scores_out=scores)
        csa.decode(d, qd, kd, vd, ptd, sld, sel, nsel, ex["prefix"], ex["window"], out, lay.ws,
                   lse, scale=1.0)
    torch.cuda.synchronize()
    assert csa.device_status(lay.ws) == 0
    if not one_call:
        for page, want in ex["expected_scores"].items():
            assert scores[0, 0, int(page)].item() == want
    assert nsel[0, 0].item() == len(ex["expected_selection"])
    assert sel[0, 0, :nsel[0, 0].item()].tolist() == ex["expected_selection"]
    o = out.float().cpu().numpy()
    # one bf16 rounding of an fp32 result
    np.testing.assert_allclose(o[0, :, :2], ex["expected_out"], rtol=2 ** -8, atol=1e-6)
    assert not o[0, :, 2:].any()
    # the probabilities enter the sum of exponentials as the bf16 values the
    # P.V product uses (each within 2^-9 relative), so lse is within ~2^-9
    np.testing.assert_allclose(lse.cpu().numpy()[0], ex["expected_lse"], rtol=1e-4, atol=1e-3)


def test_oracle_fp8_copy_on_the_worked_example():
    """Every key of the example (0, +-1, 0.5) is a power of two times an E4M3
    value, so the fp8 copy holds the exact box and its scores are the exact
    ones."""
    ex = load()
    q, k, v, pt, sl = build(ex)
    d = oracle.Dims(1, 2, 1, D, ex["page_size"], pt.shape[1], pt.shape[1])
    m8 = oracle.meta_fp8(d, oracle.meta(d, k, pt, sl), pt, sl)
    sc = oracle.scores_fp8(d, q, m8, pt, sl, ex["prefix"], ex["window"])
    for page, want in ex["expected_scores"].items():
        assert sc[0, 0, int(page)] == want


@pytest.mark.gpu
def test_cuda_fp8_path_on_the_worked_example():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_b200 import csa
    ex = load()
    q, k, v, pt, sl = build(ex)
    dev = torch.device("cuda:0")
    t = lambda a, dt: torch.from_numpy(a.astype(dt)).to(dev)
    qd = t(q, np.int16).view(torch.bfloat16)
    kd = t(k, np.int16).view(torch.bfloat16)
    vd = t(v, np.int16).view(torch.bfloat16)
    ptd, sld = t(pt, np.int32), t(sl, np.int32)
    n_pages = pt.shape[1]
    d = csa.make_dims(1, 2, 1, D, n_pages, n_pages, 4)
    lay = csa.Layer(d, kd, vd, ptd, sld, ex["prefix"], ex["window"], ex["budget"], fp8=True)
    lay.rebuild_meta()
    sel = torch.full((1, 1, 4), -7, dtype=torch.int32, device=dev)
    nsel = torch.full((1, 1), -7, dtype=torch.int32, device=dev)
    out = torch.empty((1, 2, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 2), dtype=torch.float32, device=dev)
    csa.sparse_attention_fp8(d, qd, kd, vd, lay.meta8, ptd, sld, ex["prefix"], ex["window"],
                             ex["budget"], sel, nsel, out, lay.ws, lse, scale=1.0)
    torch.cuda.synchronize()
    assert csa.device_status(lay.ws) == 0
    assert nsel[0, 0].item() == len(ex["expected_selection"])
    assert sel[0, 0, :nsel[0, 0].item()].tolist() == ex["expected_selection"]
    o = out.float().cpu().numpy()
    np.testing.assert_allclose(o[0, :, :2], ex["expected_out"], rtol=2 ** -8, atol=1e-6)
    np.testing.assert_allclose(lse.cpu().numpy()[0], ex["expected_lse"], rtol=1e-4, atol=1e-3)
