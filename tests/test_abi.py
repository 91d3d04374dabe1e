"""The C-ABI library loads, exports every symbol include/csa.h declares, and
rejects bad arguments on the host (no GPU needed: every case below returns
before any CUDA call)."""
import ctypes
import os
import re

import pytest

from long_context_decoding_b200 import build as csa_build
from long_context_decoding_b200 import csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    csa_build.build()
    return csa.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "csa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert header_functions() == sorted(csa.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert L.csa_version() == 102   # 1.02: the fp8 and context-parallel entry points
    assert csa.status_string(0) == "ok"
    assert "workspace" in csa.status_string(-3)
    assert csa.status_string(-99) == "unknown status"


def dims(**kw):
    base = dict(B=4, Hq=32, Hkv=4, D=128, max_pages_per_seq=16388, num_pages=65555, max_sel=512)
    base.update(kw)
    return csa.make_dims(**base)


def test_workspace_size_valid_and_invalid(L):
    n = csa.workspace_size(dims())
    # scores alone need B*Hkv*max_pages*4 bytes
    assert n >= 4 * 4 * 16388 * 4
    for bad in (dict(D=96), dict(Hq=12, Hkv=4), dict(Hq=30, Hkv=4), dict(B=0),
                dict(B=1024, Hkv=4, Hq=4)):
        with pytest.raises(csa.CsaError):
            csa.workspace_size(dims(**bad))
    d = dims()
    d.page_size = 32
    assert L.csa_workspace_size(ctypes.byref(d)) == 0


FAKE = ctypes.c_void_p(0x10000)        # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10008)


def test_host_validation_codes(L):
    d = dims()
    P = [FAKE] * 6
    W = (FAKE, ctypes.c_size_t(1 << 40), None)          # workspace, bytes, stream

    def score(q=FAKE, budget=64, ws=W):
        return L.csa_score_select(ctypes.byref(d), q, FAKE, FAKE, FAKE, 0, 0, budget, FAKE, FAKE,
                                  None, *ws)
    assert score(q=None) == -1                      # null pointer
    assert score(q=MISALIGNED) == -1                # not 16-byte aligned
    assert score(budget=-16) == -1                  # negative budget
    assert score(budget=16 * 513) == -1             # more pages than max_sel
    assert score(ws=(None, ctypes.c_size_t(1 << 40), None)) == -3
    assert score(ws=(FAKE, ctypes.c_size_t(16), None)) == -3
    # unsupported head dim / group size
    bad = dims(D=80)
    assert L.csa_decode_full(ctypes.byref(bad), *P[:5], ctypes.c_float(0), FAKE, None, FAKE,
                             1 << 40, None) == -2
    bad = dims(Hq=12, Hkv=4)
    assert L.csa_decode(ctypes.byref(bad), *P[:5], FAKE, FAKE, 0, 0, ctypes.c_float(0), FAKE,
                        None, FAKE, 1 << 40, None) == -2
    # sparse decode needs a selection; NaN scale is rejected
    assert L.csa_decode(ctypes.byref(d), *P[:5], None, FAKE, 0, 0, ctypes.c_float(0), FAKE, None,
                        FAKE, 1 << 40, None) == -1
    assert L.csa_decode_full(ctypes.byref(d), *P[:5], ctypes.c_float(float("nan")), FAKE, None,
                             FAKE, 1 << 40, None) == -1
    # meta update: n_new < 1, new_k without new_v
    assert L.csa_meta_update(ctypes.byref(d), *P[:5], None, None, 0, FAKE, 1 << 40, None) == -1
    assert L.csa_meta_update(ctypes.byref(d), *P[:5], FAKE, None, 1, FAKE, 1 << 40, None) == -1
    # status read without a workspace
    assert L.csa_get_device_status(None, None, None) == -3


def test_host_validation_codes_fp8_and_context_parallel(L):
    d = dims()
    W = (FAKE, ctypes.c_size_t(1 << 40), None)
    # fp8 scoring without the fp8 copy; fp8 update with a bad n_new
    assert L.csa_score_select_fp8(ctypes.byref(d), FAKE, None, FAKE, FAKE, 0, 0, 64, FAKE, FAKE,
                                  None, *W) == -1
    assert L.csa_meta_update_fp8(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                 0, *W) == -1
    # selection over given scores: null scores, budget over max_sel, no workspace
    def sel(scores=FAKE, budget=64, ws=W):
        return L.csa_select_scores(ctypes.byref(d), scores, FAKE, 0, 0, budget, FAKE, FAKE, *ws)
    assert sel(scores=None) == -1
    assert sel(scores=MISALIGNED) == -1
    assert sel(budget=16 * 513) == -1
    assert sel(ws=(FAKE, ctypes.c_size_t(16), None)) == -3
    # shard selection: an empty or inverted range is fine / rejected; max_sel_local too small
    assert L.csa_shard_selection(ctypes.byref(d), FAKE, FAKE, 10, 5, 512, FAKE, FAKE, None) == -1
    assert L.csa_shard_selection(ctypes.byref(d), FAKE, FAKE, 0, 10, 511, FAKE, FAKE, None) == -1
    assert L.csa_shard_selection(ctypes.byref(d), FAKE, None, 0, 10, 512, FAKE, FAKE, None) == -1
    # merge: parts, head_dim, pointers
    def merge(parts=2, D=128, out=FAKE):
        return L.csa_merge_attention(parts, 4, 32, D, FAKE, FAKE, out, None, None)
    assert merge(parts=0) == -1
    assert merge(parts=65) == -1
    assert merge(D=96) == -1
    assert merge(out=None) == -1
    assert merge(out=MISALIGNED) == -1


def test_binding_checks_tensor_sizes():
    """A tensor smaller than the dims say is rejected before any call (the
    kernels would run past its end)."""
    import torch
    d = dims(B=2, Hq=8, Hkv=2, D=64, max_pages_per_seq=10, num_pages=30, max_sel=4)
    csa._check_sizes(d, q=torch.empty(2 * 8 * 64), k_cache=torch.empty(30 * 2 * 16 * 64),
                     sel=torch.empty(2, 2, 4), n_sel=torch.empty(2, 2))
    for kw in (dict(q=torch.empty(2, 8, 63)), dict(k_cache=torch.empty(29, 2, 16, 64)),
               dict(meta=torch.empty(30, 2, 2, 32)), dict(page_table=torch.empty(2, 9)),
               dict(sel=torch.empty(2, 2, 3)), dict(lse=torch.empty(2, 7)),
               dict(scores_out=torch.empty(2, 2, 9)), dict(meta8=torch.empty(30, 2, 143))):
        with pytest.raises(ValueError):
            csa._check_sizes(d, **kw)
    with pytest.raises(ValueError):                  # three new tokens need 3x the rows
        csa._check_sizes(d, 3, new_k=torch.empty(2, 2, 2, 64))


def test_binding_requires_cuda_tensors():
    import torch
    d = dims(B=1, Hq=4, Hkv=1, max_pages_per_seq=4, num_pages=4, max_sel=4)
    with pytest.raises(ValueError):
        csa.decode_full(d, torch.zeros(1, 4, 128, dtype=torch.bfloat16), None, None, None, None,
                        None, torch.zeros(8, dtype=torch.uint8))
