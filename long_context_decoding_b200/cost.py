"""Algorithmic HBM bytes of one combined-sparse-attention layer step.

The decoding cost the pages' configuration search trades against accuracy
("Methodology", arxivlens analysis: "estimated decoding cost") is, for this
memory-bound decode, the bytes a step must move.  Per (sequence, kv-head)
unit with L tokens, prefix P, window W and budget:

  * metadata of the candidates: |C| pages x 4*D bytes (bf16 min + max), when
    there is a choice to make (0 < k < |C|; else no page needs a score);
  * K and V of the attended tokens:   |A| tokens x 4*D bytes;
  * q in and out: G*D*2 bytes each.

|C| counts the pages holding a token of [P', L - W') (P' = min(P, L),
W' = min(W, L)); |A| = P' + W' + the tokens the k = min(budget // 16, |C|)
selected pages add outside prefix and window.  Interior candidate pages add
16 tokens each; the two boundary pages add fewer, so |A| is bounded by the
k pages taken as interior pages (the figure used here, exact whenever the
boundary pages are not selected).  The dense layer moves L x 4*D bytes plus
q and out.  Score and split-K partial traffic stays in L2 and is not counted.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Iterable, Optional

PAGE = 16


@dataclass
class UnitBytes:
    candidates: int      # |C| pages
    k_pages: int         # pages selected
    attended: int        # |A| tokens
    meta: int            # bytes
    kv: int              # bytes


def unit_bytes(L: int, D: int, prefix: int, window: int, budget: Optional[int]) -> UnitBytes:
    Pe, We = min(prefix, L), min(window, L)
    if Pe < L - We:
        c_lo, c_hi = Pe // PAGE, -(-(L - We) // PAGE)
        n = c_hi - c_lo
        mid = L - We - Pe                     # tokens strictly between prefix and window
    else:
        n, mid = 0, 0
    k = n if budget is None else min(budget // PAGE, n)
    attended = Pe + We + min(mid, k * PAGE) if n else L
    # the metadata is read only when there is a choice to make (0 < k < |C|)
    meta = n * 4 * D if 0 < k < n else 0
    return UnitBytes(n, k, attended, meta, attended * 4 * D)


def layer_bytes(seq_lens: Iterable[int], Hq: int, Hkv: int, D: int, prefix: int, window: int,
                budget: Optional[int]) -> dict:
    """Algorithmic bytes of one sparse layer step and of the dense layer."""
    meta = kv = dense = 0
    B = 0
    for L in seq_lens:
        B += 1
        u = unit_bytes(int(L), D, prefix, window, budget)
        meta += Hkv * u.meta
        kv += Hkv * u.kv
        dense += Hkv * int(L) * 4 * D
    qo = 2 * B * Hq * D * 2
    return {"meta": meta, "kv": kv, "q_out": qo, "sparse": meta + kv + qo, "dense": dense + qo}
