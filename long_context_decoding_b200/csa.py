"""Python binding of libcsa.so (C ABI in include/csa.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libcsa.so.  Tensors are torch CUDA tensors; the calls run on the
current torch stream (or the one passed).  There is no CPU fallback: if the
library is missing or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

PAGE = 16
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_OK = 0
CSA_ERR_INVALID_ARG = -1
CSA_ERR_UNSUPPORTED = -2
CSA_ERR_WORKSPACE = -3
CSA_ERR_CUDA = -4
CSA_ERR_DEVICE_FLAG = -5
DEVFLAG_BAD_PAGE_ID = 1
DEVFLAG_BAD_SELECTION = 2
DEVFLAG_BAD_SEQ_LEN = 4
DEVFLAG_TIMEOUT = 8

EXPORTS = ("csa_version", "csa_status_string", "csa_workspace_size", "csa_workspace_init",
           "csa_meta_update", "csa_score_select", "csa_decode", "csa_decode_full",
           "csa_get_device_status", "csa_decode_noalloc", "csa_sparse_attention",
           "csa_meta_update_fp8", "csa_score_select_fp8", "csa_sparse_attention_fp8",
           "csa_select_scores", "csa_shard_selection", "csa_merge_attention")


class CsaError(RuntimeError):
    def __init__(self, where: str, status: int, msg: str):
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


class Dims(ctypes.Structure):
    """Mirror of ``csa_dims``."""

    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("page_size", ctypes.c_int),
                ("max_pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("max_sel", ctypes.c_int)]

    def __repr__(self):
        return "Dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_dims(B, Hq, Hkv, D, max_pages_per_seq, num_pages, max_sel, page_size=PAGE) -> Dims:
    return Dims(B, Hq, Hkv, D, page_size, max_pages_per_seq, num_pages, max_sel)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcsa.so (raises when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_decoding_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        D = ctypes.POINTER(Dims)
        L.csa_version.restype = I
        L.csa_status_string.argtypes = [I]
        L.csa_status_string.restype = ctypes.c_char_p
        L.csa_workspace_size.argtypes = [D]
        L.csa_workspace_size.restype = Z
        L.csa_workspace_init.argtypes = [P, Z, P]
        L.csa_meta_update.argtypes = [D, P, P, P, P, P, P, P, I, P, Z, P]
        L.csa_score_select.argtypes = [D, P, P, P, P, I, I, I, P, P, P, P, Z, P]
        L.csa_decode.argtypes = [D, P, P, P, P, P, P, P, I, I, ctypes.c_float, P, P, P, Z, P]
        L.csa_decode_full.argtypes = [D, P, P, P, P, P, ctypes.c_float, P, P, P, Z, P]
        L.csa_get_device_status.argtypes = [P, P, ctypes.POINTER(I)]
        L.csa_sparse_attention.argtypes = [D, P, P, P, P, P, P, I, I, I, ctypes.c_float, P, P, P,
                                           P, P, Z, P]
        L.csa_meta_update_fp8.argtypes = [D, P, P, P, P, P, P, P, P, I, P, Z, P]
        L.csa_score_select_fp8.argtypes = [D, P, P, P, P, I, I, I, P, P, P, P, Z, P]
        L.csa_sparse_attention_fp8.argtypes = [D, P, P, P, P, P, P, I, I, I, ctypes.c_float, P,
                                               P, P, P, P, Z, P]
        L.csa_select_scores.argtypes = [D, P, P, I, I, I, P, P, P, Z, P]
        L.csa_shard_selection.argtypes = [D, P, P, I, I, I, P, P, P]
        L.csa_merge_attention.argtypes = [I, I, I, I, P, P, P, P, P]
        for f in ("csa_workspace_init", "csa_meta_update", "csa_score_select", "csa_decode",
                  "csa_decode_full", "csa_get_device_status", "csa_sparse_attention",
                  "csa_meta_update_fp8", "csa_score_select_fp8", "csa_sparse_attention_fp8",
                  "csa_select_scores", "csa_shard_selection", "csa_merge_attention"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().csa_status_string(int(st)).decode()


def _check(where: str, st: int):
    if st != CSA_OK:
        raise CsaError(where, st, status_string(st))


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _sizes(d: Dims, n_new: int = 1) -> dict:
    """Elements each named argument of dims d must hold, at least (the C
    calls index them by d's sizes)."""
    B, Hq, Hkv, D = d.B, d.Hq, d.Hkv, d.D
    NPG, MP = d.num_pages, d.max_pages_per_seq
    return {"q": B * Hq * D, "out": B * Hq * D, "lse": B * Hq,
            "k_cache": NPG * Hkv * 16 * D, "v_cache": NPG * Hkv * 16 * D,
            "meta": NPG * Hkv * 2 * D, "meta8": NPG * Hkv * (2 * D + 16),
            "page_table": B * MP, "seq_lens": B, "sel": B * Hkv * d.max_sel, "n_sel": B * Hkv,
            "scores": B * Hkv * MP, "scores_out": B * Hkv * MP,
            "new_k": B * n_new * Hkv * D, "new_v": B * n_new * Hkv * D}


def _check_sizes(d: Dims, n_new: int = 1, **tensors):
    """Raise ValueError when a tensor is smaller than dims d require: a call
    would read or write past its end."""
    need = _sizes(d, max(1, int(n_new)))
    for name, t in tensors.items():
        if t is not None and t.numel() < need[name]:
            raise ValueError(f"{name} holds {t.numel()} elements; dims need {need[name]}")


def workspace_size(d: Dims) -> int:
    n = lib().csa_workspace_size(ctypes.byref(d))
    if n == 0:
        raise CsaError("csa_workspace_size", -2, "invalid or unsupported shape")
    return int(n)


def new_workspace(d: Dims, device="cuda", stream=None) -> torch.Tensor:
    """Allocate (with torch) and zero a workspace for shape ``d``."""
    ws = torch.empty(workspace_size(d), dtype=torch.uint8, device=device)
    _check("csa_workspace_init",
           lib().csa_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))
    return ws


def meta_update(d: Dims, k_cache, v_cache, meta, page_table, seq_lens, new_k, new_v, n_new: int,
                ws, stream=None):
    """Append n_new tokens per sequence (new_k/new_v None: rebuild metadata)."""
    _check_sizes(d, n_new, k_cache=k_cache, v_cache=v_cache, meta=meta, page_table=page_table,
                 seq_lens=seq_lens, new_k=new_k, new_v=new_v)
    bf = torch.bfloat16
    _check("csa_meta_update", lib().csa_meta_update(
        ctypes.byref(d), _ptr(k_cache, bf, "k_cache"), _ptr(v_cache, bf, "v_cache"),
        _ptr(meta, bf, "meta"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(new_k, bf, "new_k"),
        _ptr(new_v, bf, "new_v"), int(n_new), _ptr(ws), ws.numel(), _stream(stream)))


def score_select(d: Dims, q, meta, page_table, seq_lens, prefix: int, window: int, budget: int,
                 sel, n_sel, ws, scores_out=None, stream=None):
    """Quest scores from metadata and top-k page selection into sel / n_sel."""
    _check_sizes(d, q=q, meta=meta, page_table=page_table, seq_lens=seq_lens, sel=sel,
                 n_sel=n_sel, scores_out=scores_out)
    bf = torch.bfloat16
    _check("csa_score_select", lib().csa_score_select(
        ctypes.byref(d), _ptr(q, bf, "q"), _ptr(meta, bf, "meta"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        int(prefix), int(window), int(budget), _ptr(sel, torch.int32, "sel"),
        _ptr(n_sel, torch.int32, "n_sel"), _ptr(scores_out, torch.float32, "scores_out"),
        _ptr(ws), ws.numel(), _stream(stream)))


def decode(d: Dims, q, k_cache, v_cache, page_table, seq_lens, sel, n_sel, prefix: int,
           window: int, out, ws, lse=None, scale: float = 0.0, stream=None):
    """Combined sparse attention over prefix + window + selected pages."""
    _check_sizes(d, q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table,
                 seq_lens=seq_lens, sel=sel, n_sel=n_sel, out=out, lse=lse)
    bf = torch.bfloat16
    _check("csa_decode", lib().csa_decode(
        ctypes.byref(d), _ptr(q, bf, "q"), _ptr(k_cache, bf, "k_cache"),
        _ptr(v_cache, bf, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(sel, torch.int32, "sel"),
        _ptr(n_sel, torch.int32, "n_sel"), int(prefix), int(window), float(scale),
        _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"), _ptr(ws), ws.numel(),
        _stream(stream)))


def sparse_attention(d: Dims, q, k_cache, v_cache, meta, page_table, seq_lens, prefix: int,
                     window: int, budget: int, sel, n_sel, out, ws, lse=None, scale: float = 0.0,
                     stream=None):
    """Scoring, top-k selection and the sparse decode in one call (the
    selection and the decode of the selected pages share a launch when the
    shape allows)."""
    _check_sizes(d, q=q, k_cache=k_cache, v_cache=v_cache, meta=meta, page_table=page_table,
                 seq_lens=seq_lens, sel=sel, n_sel=n_sel, out=out, lse=lse)
    bf = torch.bfloat16
    _check("csa_sparse_attention", lib().csa_sparse_attention(
        ctypes.byref(d), _ptr(q, bf, "q"), _ptr(k_cache, bf, "k_cache"),
        _ptr(v_cache, bf, "v_cache"), _ptr(meta, bf, "meta"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        int(prefix), int(window), int(budget), float(scale), _ptr(sel, torch.int32, "sel"),
        _ptr(n_sel, torch.int32, "n_sel"), _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(ws), ws.numel(), _stream(stream)))


def select_scores(d: Dims, scores, seq_lens, prefix: int, window: int, budget: int, sel, n_sel,
                  ws, stream=None):
    """Top-k pages over given fp32 scores [B][Hkv][max_pages_per_seq] (the
    selection csa_score_select makes from its own scores)."""
    _check_sizes(d, scores=scores, seq_lens=seq_lens, sel=sel, n_sel=n_sel)
    _check("csa_select_scores", lib().csa_select_scores(
        ctypes.byref(d), _ptr(scores, torch.float32, "scores"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(prefix), int(window), int(budget),
        _ptr(sel, torch.int32, "sel"), _ptr(n_sel, torch.int32, "n_sel"), _ptr(ws), ws.numel(),
        _stream(stream)))


def shard_selection(d: Dims, sel, n_sel, page_lo: int, page_hi: int, sel_local, n_sel_local,
                    stream=None):
    """The selected pages in [page_lo, page_hi), as pages of that shard."""
    _check_sizes(d, sel=sel, n_sel=n_sel)
    if sel_local.numel() < d.B * d.Hkv * sel_local.shape[-1] or n_sel_local.numel() < d.B * d.Hkv:
        raise ValueError("sel_local / n_sel_local smaller than [B][Hkv][...]")
    _check("csa_shard_selection", lib().csa_shard_selection(
        ctypes.byref(d), _ptr(sel, torch.int32, "sel"), _ptr(n_sel, torch.int32, "n_sel"),
        int(page_lo), int(page_hi), int(sel_local.shape[-1]),
        _ptr(sel_local, torch.int32, "sel_local"), _ptr(n_sel_local, torch.int32, "n_sel_local"),
        _stream(stream)))


def merge_attention(out_parts, lse_parts, out, lse=None, stream=None):
    """Log-sum-exp merge of partial attentions over disjoint token sets:
    out_parts bf16 [R][B][Hq][D], lse_parts fp32 [R][B][Hq]."""
    R, B, Hq, D = out_parts.shape
    if lse_parts.numel() < R * B * Hq or out.numel() < B * Hq * D or \
            (lse is not None and lse.numel() < B * Hq):
        raise ValueError("lse_parts [R][B][Hq], out [B][Hq][D] and lse [B][Hq] must match out_parts")
    _check("csa_merge_attention", lib().csa_merge_attention(
        int(R), int(B), int(Hq), int(D), _ptr(out_parts, torch.bfloat16, "out_parts"),
        _ptr(lse_parts, torch.float32, "lse_parts"), _ptr(out, torch.bfloat16, "out"),
        _ptr(lse, torch.float32, "lse"), _stream(stream)))


def meta8_row_bytes(D: int) -> int:
    """Bytes of one (page, kv-head) row of the fp8 metadata copy."""
    return 2 * D + 16


def new_meta8(d: Dims, device="cuda") -> torch.Tensor:
    """fp8 metadata copy, uint8 [num_pages][Hkv][2*D + 16]."""
    return torch.zeros((d.num_pages, d.Hkv, meta8_row_bytes(d.D)), dtype=torch.uint8,
                       device=device)


def meta_update_fp8(d: Dims, k_cache, v_cache, meta, meta8, page_table, seq_lens, new_k, new_v,
                    n_new: int, ws, stream=None):
    """csa_meta_update that also keeps the fp8 copy meta8 current."""
    _check_sizes(d, n_new, k_cache=k_cache, v_cache=v_cache, meta=meta, meta8=meta8,
                 page_table=page_table, seq_lens=seq_lens, new_k=new_k, new_v=new_v)
    bf = torch.bfloat16
    _check("csa_meta_update_fp8", lib().csa_meta_update_fp8(
        ctypes.byref(d), _ptr(k_cache, bf, "k_cache"), _ptr(v_cache, bf, "v_cache"),
        _ptr(meta, bf, "meta"), _ptr(meta8, torch.uint8, "meta8"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(new_k, bf, "new_k"), _ptr(new_v, bf, "new_v"), int(n_new), _ptr(ws), ws.numel(),
        _stream(stream)))


def score_select_fp8(d: Dims, q, meta8, page_table, seq_lens, prefix: int, window: int,
                     budget: int, sel, n_sel, ws, scores_out=None, stream=None):
    """csa_score_select with the scores from the fp8 metadata copy."""
    _check_sizes(d, q=q, meta8=meta8, page_table=page_table, seq_lens=seq_lens, sel=sel,
                 n_sel=n_sel, scores_out=scores_out)
    _check("csa_score_select_fp8", lib().csa_score_select_fp8(
        ctypes.byref(d), _ptr(q, torch.bfloat16, "q"), _ptr(meta8, torch.uint8, "meta8"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        int(prefix), int(window), int(budget), _ptr(sel, torch.int32, "sel"),
        _ptr(n_sel, torch.int32, "n_sel"), _ptr(scores_out, torch.float32, "scores_out"),
        _ptr(ws), ws.numel(), _stream(stream)))


def sparse_attention_fp8(d: Dims, q, k_cache, v_cache, meta8, page_table, seq_lens,
                         prefix: int, window: int, budget: int, sel, n_sel, out, ws, lse=None,
                         scale: float = 0.0, stream=None):
    """csa_sparse_attention with the scores from the fp8 metadata copy."""
    _check_sizes(d, q=q, k_cache=k_cache, v_cache=v_cache, meta8=meta8, page_table=page_table,
                 seq_lens=seq_lens, sel=sel, n_sel=n_sel, out=out, lse=lse)
    bf = torch.bfloat16
    _check("csa_sparse_attention_fp8", lib().csa_sparse_attention_fp8(
        ctypes.byref(d), _ptr(q, bf, "q"), _ptr(k_cache, bf, "k_cache"),
        _ptr(v_cache, bf, "v_cache"), _ptr(meta8, torch.uint8, "meta8"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        int(prefix), int(window), int(budget), float(scale), _ptr(sel, torch.int32, "sel"),
        _ptr(n_sel, torch.int32, "n_sel"), _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(ws), ws.numel(), _stream(stream)))


def decode_full(d: Dims, q, k_cache, v_cache, page_table, seq_lens, out, ws, lse=None,
                scale: float = 0.0, stream=None):
    """Dense decode over every valid token (the unmodified layer)."""
    _check_sizes(d, q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table,
                 seq_lens=seq_lens, out=out, lse=lse)
    bf = torch.bfloat16
    _check("csa_decode_full", lib().csa_decode_full(
        ctypes.byref(d), _ptr(q, bf, "q"), _ptr(k_cache, bf, "k_cache"),
        _ptr(v_cache, bf, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), float(scale), _ptr(out, bf, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(ws), ws.numel(), _stream(stream)))


def decode_noalloc(d: Dims, q, k_cache, v_cache, page_table, seq_lens, sel, n_sel, prefix: int,
                   window: int, out, lse=None, scale: float = 0.0, stream=None):
    """csa_decode without a workspace, for callers that cannot allocate device
    memory (a plugin inside a runtime that owns all device buffers, a server
    that reserves the GPU at start-up): the scratch is a fixed 8 MiB array
    inside the library, shared by every call on the device, so calls must
    not overlap on the GPU.  Device-side flags of this call are not
    reported."""
    _check_sizes(d, q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table,
                 seq_lens=seq_lens, sel=sel, n_sel=n_sel, out=out, lse=lse)
    f = lib().csa_decode_noalloc
    P = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(Dims), P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                  ctypes.c_float, P, P, P]
    f.restype = ctypes.c_int
    bf = torch.bfloat16
    _check("csa_decode_noalloc", f(
        ctypes.byref(d), _ptr(q, bf, "q"), _ptr(k_cache, bf, "k_cache"),
        _ptr(v_cache, bf, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(sel, torch.int32, "sel"),
        _ptr(n_sel, torch.int32, "n_sel"), int(prefix), int(window), float(scale),
        _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"), _stream(stream)))


def device_status(ws, stream=None) -> int:
    """Synchronise, return and clear the device flag bits (0 = clean)."""
    flags = ctypes.c_int(0)
    st = lib().csa_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(flags))
    if st not in (CSA_OK, CSA_ERR_DEVICE_FLAG):
        _check("csa_get_device_status", st)
    return int(flags.value)


class Layer:
    """Device state of one full-attention layer: a paged cache, its page
    metadata, the page table, sequence lengths and the per-layer
    (prefix, window, budget).  ``step`` runs one decode step through the
    C ABI: append + metadata update, score + select, sparse decode."""

    def __init__(self, d: Dims, k_cache, v_cache, page_table, seq_lens, prefix: int, window: int,
                 budget: int, meta=None, ws=None, fp8: bool = False):
        self.d = d
        dev = k_cache.device
        self.k_cache, self.v_cache = k_cache, v_cache
        self.page_table, self.seq_lens = page_table, seq_lens
        self.prefix, self.window, self.budget = prefix, window, budget
        self.meta = meta if meta is not None else torch.zeros(
            (d.num_pages, d.Hkv, 2, d.D), dtype=torch.bfloat16, device=dev)
        self.ws = ws if ws is not None else new_workspace(d, dev)
        # fp8: also keep the fp8 metadata copy and score from it
        self.meta8 = new_meta8(d, dev) if fp8 else None
        self.sel = torch.zeros((d.B, d.Hkv, d.max_sel), dtype=torch.int32, device=dev)
        self.n_sel = torch.zeros((d.B, d.Hkv), dtype=torch.int32, device=dev)
        self.out = torch.empty((d.B, d.Hq, d.D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((d.B, d.Hq), dtype=torch.float32, device=dev)

    def rebuild_meta(self, stream=None):
        n = self.d.max_pages_per_seq * PAGE
        if self.meta8 is not None:
            meta_update_fp8(self.d, self.k_cache, self.v_cache, self.meta, self.meta8,
                            self.page_table, self.seq_lens, None, None, n, self.ws, stream)
            return
        meta_update(self.d, self.k_cache, self.v_cache, self.meta, self.page_table, self.seq_lens,
                    None, None, n, self.ws, stream)

    def step(self, q, new_k=None, new_v=None, stream=None, fused=False):
        """One decode step.  With new_k/new_v ([B][1][Hkv][D]) the token is
        appended first; seq_lens must already count it.  fused=True runs
        scoring, selection and decode as one csa_sparse_attention call."""
        if self.meta8 is not None:
            if new_k is not None:
                meta_update_fp8(self.d, self.k_cache, self.v_cache, self.meta, self.meta8,
                                self.page_table, self.seq_lens, new_k, new_v, new_k.shape[1],
                                self.ws, stream)
            if fused:
                sparse_attention_fp8(self.d, q, self.k_cache, self.v_cache, self.meta8,
                                     self.page_table, self.seq_lens, self.prefix, self.window,
                                     self.budget, self.sel, self.n_sel, self.out, self.ws,
                                     self.lse, stream=stream)
            else:
                score_select_fp8(self.d, q, self.meta8, self.page_table, self.seq_lens,
                                 self.prefix, self.window, self.budget, self.sel, self.n_sel,
                                 self.ws, stream=stream)
                decode(self.d, q, self.k_cache, self.v_cache, self.page_table, self.seq_lens,
                       self.sel, self.n_sel, self.prefix, self.window, self.out, self.ws,
                       self.lse, stream=stream)
            return self.out
        if new_k is not None:
            meta_update(self.d, self.k_cache, self.v_cache, self.meta, self.page_table,
                        self.seq_lens, new_k, new_v, new_k.shape[1], self.ws, stream)
        if fused:
            sparse_attention(self.d, q, self.k_cache, self.v_cache, self.meta, self.page_table,
                             self.seq_lens, self.prefix, self.window, self.budget, self.sel,
                             self.n_sel, self.out, self.ws, self.lse, stream=stream)
            return self.out
        score_select(self.d, q, self.meta, self.page_table, self.seq_lens, self.prefix,
                     self.window, self.budget, self.sel, self.n_sel, self.ws, stream=stream)
        decode(self.d, q, self.k_cache, self.v_cache, self.page_table, self.seq_lens, self.sel,
               self.n_sel, self.prefix, self.window, self.out, self.ws, self.lse, stream=stream)
        return self.out
