"""Seeded synthetic inputs for combined sparse decode attention.

This module only draws random inputs and lays them out in the paged-cache
format; it holds none of the method's arithmetic (no scoring, selection or
attention).  It is the one module that both the CUDA path (tests, bench)
and the CPU oracle (tests) take their inputs from.

The shapes stand in for the batch-4, 64k/256k-token decode workload that the
roboaidigest post ("What It Buys") quotes the speedups on; the pages'
21 long-context datasets and trained weights are not used (no data or
weights are available), so q, K and V are Gaussian draws with the structure
each workload names (per-channel key outliers, planted q-aligned pages,
ragged lengths).

Cache recipe, every workload:
  * physical pages are a seeded random permutation of the pool, so the
    page-table indirection is real; the pool has a few spare pages;
  * every slot beyond a sequence's length, and every page no sequence
    owns, is poisoned with NaN so that a kernel reading one shows it;
  * generation order: q, K, V, then outlier scales / plants, then the page
    permutation, all from one ``torch.Generator`` seeded per workload (and
    per layer), on the device the tensors are made on.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional, Sequence, Tuple

import torch

PAGE = 16
BF16_NAN = 0x7FC0


@dataclass(frozen=True)
class Workload:
    """One decode-attention workload (one layer unless ``layers`` > 1)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    seq_lens: Tuple[int, ...]       # per sequence, before any appended step
    prefix: int
    window: int
    budget: int
    seed: int = 0
    k_outlier: bool = False         # K *= LogNormal(0,1) per (kv-head, channel)
    planted: int = 0                # q-aligned planted pages per (seq, kv-head)
    layers: int = 1
    layer_cfgs: Tuple[Tuple[int, int], ...] = ()   # per-layer (window, budget) cycle
    steps: int = 0                  # decode steps with append (capacity is reserved)
    spare_pages: int = 3

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def layer_window_budget(self, layer: int) -> Tuple[int, int]:
        if self.layer_cfgs:
            return self.layer_cfgs[layer % len(self.layer_cfgs)]
        return self.window, self.budget

    @property
    def max_pages(self) -> int:
        return -(-(max(self.seq_lens) + self.steps) // PAGE)

    @property
    def num_pages(self) -> int:
        return self.B * self.max_pages + self.spare_pages

    @property
    def max_sel(self) -> int:
        budgets = [b for _, b in self.layer_cfgs] or [self.budget]
        return max(1, max(budgets) // PAGE)


def _ragged(B: int, lo: int, hi: int, seed: int) -> Tuple[int, ...]:
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g))


# The five workloads, smallest first.
TINY = Workload("b1_h4x1_d128_ctx4k", B=1, Hq=4, Hkv=1, D=128, seq_lens=(4096,),
                prefix=64, window=256, budget=512)
CTX32K = Workload("b4_h16x4_d128_ctx32k_outlier", B=4, Hq=16, Hkv=4, D=128,
                  seq_lens=(32768,) * 4, prefix=128, window=1024, budget=2048,
                  k_outlier=True)
CTX64K = Workload("b4_h16x2_d256_ctx64k_planted", B=4, Hq=16, Hkv=2, D=256,
                  seq_lens=(65536,) * 4, prefix=128, window=2048, budget=4096,
                  planted=32)
CTX256K = Workload("b4_h32x4_d128_ctx256k_12layer", B=4, Hq=32, Hkv=4, D=128,
                   seq_lens=(262144,) * 4, prefix=128, window=512, budget=1024,
                   layers=12,
                   layer_cfgs=((512, 1024), (1024, 2048), (2048, 4096), (4096, 8192)),
                   steps=64)
SWEEP = Workload("b4_h16x4_d128_ragged4k_256k", B=4, Hq=16, Hkv=4, D=128,
                 seq_lens=_ragged(4, 4096, 262144, 0), prefix=128, window=1024,
                 budget=4096)
# A larger batch of the 64k decode (another size of the model family): 8
# sequences x 8 kv-heads = 64 (sequence, kv-head) units, D = 128.
CTX64K_B8 = Workload("b8_h64x8_d128_ctx64k", B=8, Hq=64, Hkv=8, D=128,
                     seq_lens=(65536,) * 8, prefix=128, window=2048, budget=4096)
SWEEP_BUDGETS = (0, 1024, 4096, None)      # None = the whole context ("all")
SWEEP_GRID = (4096, 8192, 16384, 32768, 65536, 131072, 262144)

WORKLOADS = {w.name: w for w in (TINY, CTX32K, CTX64K, CTX256K, SWEEP, CTX64K_B8)}


@dataclass
class Case:
    """Device (or host) tensors of one layer of a workload."""

    w: Workload
    layer: int
    q: torch.Tensor            # bf16 [B][Hq][D]
    k_cache: torch.Tensor      # bf16 [num_pages][Hkv][16][D]
    v_cache: torch.Tensor
    page_table: torch.Tensor   # int32 [B][max_pages]
    seq_lens: torch.Tensor     # int32 [B]
    window: int
    budget: int
    planted_pages: Optional[torch.Tensor] = None   # int64 [B][Hkv][planted]
    gen: Optional[torch.Generator] = field(default=None, repr=False)

    @property
    def prefix(self) -> int:
        return self.w.prefix


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_case(w: Workload, device="cpu", layer: int = 0, poison: bool = True,
              seq_lens: Optional[Sequence[int]] = None) -> Case:
    """Draw one layer of workload ``w`` on ``device``.

    ``seq_lens`` overrides the workload's lengths (they must fit its page
    capacity)."""
    device = torch.device(device)
    lens = tuple(seq_lens) if seq_lens is not None else w.seq_lens
    assert len(lens) == w.B and max(lens) <= w.max_pages * PAGE
    g = _generator(device, w.seed * 1000 + layer)
    bf16 = torch.bfloat16
    q = torch.randn((w.B, w.Hq, w.D), generator=g, device=device, dtype=torch.float32).to(bf16)
    k = torch.randn((w.num_pages, w.Hkv, PAGE, w.D), generator=g, device=device, dtype=bf16)
    v = torch.randn((w.num_pages, w.Hkv, PAGE, w.D), generator=g, device=device, dtype=bf16)
    if w.k_outlier:
        c = torch.randn((w.Hkv, w.D), generator=g, device=device, dtype=torch.float32).exp_()
        k.mul_(c.to(bf16).view(1, w.Hkv, 1, w.D))
    perm = torch.randperm(w.num_pages, generator=g, device=device)
    page_table = perm[: w.B * w.max_pages].view(w.B, w.max_pages).to(torch.int32).contiguous()
    seq = torch.tensor(lens, dtype=torch.int32, device=device)
    planted = None
    if w.planted:
        planted = _plant(w, q, k, page_table, lens, g)
    window, budget = w.layer_window_budget(layer)
    case = Case(w, layer, q, k, v, page_table, seq, window, budget, planted, g)
    if poison:
        poison_unused(case)
    return case


def _plant(w: Workload, q, k, page_table, lens, g) -> torch.Tensor:
    """Overwrite ``w.planted`` pages per (sequence, kv-head) with keys
    3 * q_hat + N(0, 1), q_hat = unit vector along the sum of the group's
    queries.  Pages are drawn uniformly from the logical pages that lie
    wholly between the prefix and the window."""
    out = torch.empty((w.B, w.Hkv, w.planted), dtype=torch.int64, device=q.device)
    for b in range(w.B):
        lo = -(-w.prefix // PAGE)
        hi = (lens[b] - w.window) // PAGE
        assert hi - lo >= w.planted, "not enough pages to plant"
        for gk in range(w.Hkv):
            grp = q[b, gk * w.G:(gk + 1) * w.G].float().sum(0)
            qhat = grp / grp.norm()
            pick = torch.randperm(hi - lo, generator=g, device=q.device)[: w.planted] + lo
            out[b, gk] = pick
            noise = torch.randn((w.planted, PAGE, w.D), generator=g, device=q.device)
            keys = (3.0 * qhat).view(1, 1, w.D) + noise
            phys = page_table[b, pick].long()
            k[phys, gk] = keys.to(k.dtype)
    return out


def poison_unused(case: Case) -> None:
    """NaN-fill every slot at or beyond a sequence's length and every
    physical page no sequence owns (tracks ``case.seq_lens``)."""
    w = case.w
    nan = torch.tensor(BF16_NAN, dtype=torch.int16, device=case.k_cache.device)
    owned = torch.zeros(w.num_pages, dtype=torch.bool, device=case.k_cache.device)
    owned[case.page_table.flatten().long()] = True
    kv = (case.k_cache.view(torch.int16), case.v_cache.view(torch.int16))
    for t in kv:
        t[~owned] = nan
    lens = case.seq_lens.tolist()
    for b in range(w.B):
        L = lens[b]
        first = L // PAGE
        if L % PAGE:
            phys = int(case.page_table[b, first])
            for t in kv:
                t[phys, :, L % PAGE:, :] = nan
            first += 1
        if first < w.max_pages:
            phys = case.page_table[b, first:].long()
            for t in kv:
                t[phys] = nan


def step_tokens(case: Case, step: int, n_new: int = 1):
    """q, new_k, new_v of decode step ``step`` (bf16: [B][Hq][D] and
    [B][n_new][Hkv][D]), drawn from their own seeded generator."""
    w = case.w
    dev = case.q.device
    g = _generator(dev, 7919 + w.seed * 1000003 + case.layer * 10007 + step)
    q = torch.randn((w.B, w.Hq, w.D), generator=g, device=dev).to(torch.bfloat16)
    nk = torch.randn((w.B, n_new, w.Hkv, w.D), generator=g, device=dev).to(torch.bfloat16)
    nv = torch.randn((w.B, n_new, w.Hkv, w.D), generator=g, device=dev).to(torch.bfloat16)
    return q, nk, nv


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its raw bits (host copy)."""
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dims_tuple(w: Workload):
    """(B, Hq, Hkv, D, page_size, max_pages_per_seq, num_pages, max_sel)."""
    return (w.B, w.Hq, w.Hkv, w.D, PAGE, w.max_pages, w.num_pages, w.max_sel)


def small(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (for reduced test sizes)."""
    return replace(w, **kw)
