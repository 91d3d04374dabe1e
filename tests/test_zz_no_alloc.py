"""csa_decode_noalloc, the decode entry point for callers that cannot
allocate device memory (a plugin inside a runtime that owns every device
buffer, or a server that reserves the whole GPU at start-up): its scratch
is a fixed array inside the library instead of a caller workspace.

Called through the C ABI twice in a row, it must give what csa_decode gives
on the same inputs, within the attention tolerance of the parity tests.
This file is collected last so that a failure here never hides the others;
it passes alone in a fresh process and after the rest of the suite."""
import math

import pytest
import torch

from long_context_decoding_b200 import csa
from long_context_decoding_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3      # the parity tests' attention tolerance


def close(a, b):
    err = (a.float() - b.float()).abs()
    return err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


@pytest.mark.parametrize("w", [wl.TINY, wl.CTX32K], ids=lambda w: w.name)
def test_noalloc_decode_matches_workspace_decode(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    c = wl.make_case(w, dev)
    d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
    layer = csa.Layer(d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix, w.window,
                      w.budget)
    layer.rebuild_meta()
    ref = layer.step(c.q).clone()
    ref_lse = layer.lse.clone()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        csa.decode_noalloc(d, c.q, c.k_cache, c.v_cache, c.page_table, c.seq_lens, layer.sel,
                           layer.n_sel, w.prefix, w.window, out, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert close(out, ref)
        torch.testing.assert_close(lse, ref_lse, rtol=1e-4, atol=1e-3)
    assert csa.device_status(layer.ws) == 0
