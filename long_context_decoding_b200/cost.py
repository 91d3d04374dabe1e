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


def path_of(L: int, prefix: int, window: int, budget) -> str:
    """Which kernels a csa_sparse_attention call runs for a sequence of L
    tokens: the prefix/window decode alone (no page to select), the dense
    decode (every candidate kept: budget "all" or k >= the candidates) or
    the one-call path (scoring, fused selection + attention, combine)."""
    if budget is None or budget == "all":
        return "dense"
    u = unit_bytes(int(L), 1, prefix, window, int(budget))
    if u.k_pages == 0:
        return "prefix_window"
    return "dense" if u.k_pages >= u.candidates else "one_call"


def fit_per_path(points) -> dict:
    """t = t0[path] + bytes / bw: one bandwidth, one fixed cost per path,
    fitted by least squares on the relative error (weights 1 / t^2, so that
    the short calls count as much as the long ones).  points: dicts with
    "path" (path_of), "sparse_bytes", "sparse_us"."""
    groups = {}
    for p in points:
        groups.setdefault(p["path"], []).append(
            (float(p["sparse_bytes"]), float(p["sparse_us"]) * 1e-6))
    # within each path: weighted means; then the shared slope
    stats = {}
    num = den = 0.0
    for k, g in groups.items():
        w = [1.0 / (y * y) for _, y in g]
        sw = sum(w)
        mx = sum(wi * x for wi, (x, _) in zip(w, g)) / sw
        my = sum(wi * y for wi, (_, y) in zip(w, g)) / sw
        stats[k] = (mx, my)
        num += sum(wi * (x - mx) * (y - my) for wi, (x, y) in zip(w, g))
        den += sum(wi * (x - mx) ** 2 for wi, (x, _) in zip(w, g))
    slope = num / den
    t0 = {k: my - slope * mx for k, (mx, my) in stats.items()}
    worst = max(abs(t0[p["path"]] + slope * float(p["sparse_bytes"])
                    - float(p["sparse_us"]) * 1e-6) / (float(p["sparse_us"]) * 1e-6)
                for p in points)
    return {"bw_gbs": 1.0 / slope / 1e9, "t0_us": {k: 1e6 * v for k, v in t0.items()},
            "max_rel_err": worst,
            "form": "t = t0[path] + algorithmic bytes / bw (least squares on relative error)"}
