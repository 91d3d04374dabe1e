"""Context parallelism: one layer's decode step with every sequence's pages
split over R ranks (one process per GPU), with one exchange step.

Combined sparse attention ("Accelerating Long-Context Decoding in
Large-Scale Hybrid LLMs Without Retraining", abstract; "Methodology" on the
arxivlens page) attends each query head to the prefix, the window and the
query-aware top-k pages of the full cache.  Split by pages:

  1. every rank scores its own candidate pages (``csa_score_select`` with
     budget 0 and a score output; rank 0 holds the prefix, the last rank the
     window, so the ranks' candidates are exactly the global ones);
  2. the ranks all-gather the score arrays; concatenated along the page axis
     they are the single-GPU scores, and every rank selects the same global
     top-k from them (``csa_select_scores``: exact, ties to the lower page);
  3. every rank keeps the selected pages it holds (``csa_shard_selection``)
     and attends over them and its share of prefix and window
     (``csa_decode``);
  4. the ranks all-gather (out, lse) and merge them (``csa_merge_attention``):
     the attention over a union of disjoint token sets is the log-sum-exp
     merge of the attentions over the parts.

The bytes exchanged per unit are the shard's candidate scores (4 bytes a
page) and G (D + 1) values of the partial result.  Every arithmetic step runs
in the library's kernels; this module is host logic: the page split, the
per-rank geometry and the order of the calls and collectives.
"""
from dataclasses import dataclass
from typing import List, Sequence

import torch

from . import csa

PAGE = 16


@dataclass(frozen=True)
class ShardPlan:
    """Page boundaries 0 = p_0 < p_1 < ... < p_R = max_pages: rank r holds the
    logical pages [p_r, p_{r+1}) of every sequence."""
    splits: tuple

    @property
    def world(self) -> int:
        return len(self.splits) - 1

    def lo(self, r: int) -> int:
        return self.splits[r]

    def hi(self, r: int) -> int:
        return self.splits[r + 1]

    def local_seq_lens(self, seq_lens: Sequence[int], r: int) -> List[int]:
        """Tokens of each sequence in rank r's pages."""
        a, b = PAGE * self.lo(r), PAGE * self.hi(r)
        return [max(0, min(int(L), b) - a) for L in seq_lens]

    def local_prefix_window(self, r: int, prefix: int, window: int):
        """(prefix, window) of rank r's shard: the prefix lies in rank 0's
        pages and the window in the last rank's (plan_shards checks it)."""
        return (prefix if r == 0 else 0), (window if r == self.world - 1 else 0)


def plan_shards(max_pages: int, world: int, prefix: int, window: int,
                seq_lens: Sequence[int]) -> ShardPlan:
    """An even split of the page axis over `world` ranks.  Raises ValueError
    unless every rank gets at least one page, rank 0 holds every sequence's
    prefix tokens and the last rank every sequence's window tokens (the
    per-rank prefix and window arguments are then rank 0's prefix and the
    last rank's window, and every other rank's pages are candidates only)."""
    if world < 1 or max_pages < world:
        raise ValueError("every rank needs at least one page")
    splits = tuple(max_pages * r // world for r in range(world + 1))
    plan = ShardPlan(splits)
    for L in seq_lens:
        L = int(L)
        pe, we = min(prefix, L), min(window, L)
        if world > 1 and pe > PAGE * plan.hi(0):
            raise ValueError(f"the prefix of a {L}-token sequence spills past rank 0's pages")
        if world > 1 and L - we < PAGE * plan.lo(world - 1):
            raise ValueError(f"the window of a {L}-token sequence starts before the last "
                             "rank's pages")
    return plan


class TorchExchange:
    """all_gather over a torch.distributed process group (NCCL between
    GPUs; gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    def all_gather(self, t: torch.Tensor) -> List[torch.Tensor]:
        out = [torch.empty_like(t) for _ in range(self.dist.get_world_size(self.group))]
        self.dist.all_gather(out, t.contiguous(), group=self.group)
        return out


@dataclass
class Shard:
    """Rank r's share of one layer: its pages of every sequence in its own
    cache (page_table [B][p_{r+1} - p_r] into k_cache/v_cache/meta)."""
    rank: int
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    meta: torch.Tensor
    page_table: torch.Tensor
    seq_lens: torch.Tensor          # int32 [B]: this shard's tokens of each sequence


class CudaOps:
    """The four steps of a rank on its GPU, through the C ABI."""

    def __init__(self, plan: ShardPlan, d_global: csa.Dims, shard: Shard, seq_lens_global,
                 prefix: int, window: int, budget: int, scale: float = 0.0):
        r = shard.rank
        dev = shard.k_cache.device
        self.plan, self.sh = plan, shard
        self.dg = d_global
        self.lo, self.hi = plan.lo(r), plan.hi(r)
        self.dl = csa.make_dims(d_global.B, d_global.Hq, d_global.Hkv, d_global.D,
                                self.hi - self.lo, int(shard.k_cache.shape[0]),
                                d_global.max_sel)
        self.P, self.W = prefix, window
        self.Pr, self.Wr = plan.local_prefix_window(r, prefix, window)
        self.budget, self.scale = budget, scale
        self.sl_global = seq_lens_global
        self.ws_local = csa.new_workspace(self.dl, dev)
        self.ws_global = csa.new_workspace(self.dg, dev)
        B, Hkv, Hq, D = self.dg.B, self.dg.Hkv, self.dg.Hq, self.dg.D
        self.scores = torch.full((B, Hkv, self.hi - self.lo), float("-inf"), device=dev)
        self.sel_tmp = torch.zeros((B, Hkv, self.dl.max_sel), dtype=torch.int32, device=dev)
        self.nsel_tmp = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
        self.sel = torch.zeros_like(self.sel_tmp)
        self.n_sel = torch.zeros_like(self.nsel_tmp)
        self.sel_local = torch.zeros_like(self.sel_tmp)
        self.n_local = torch.zeros_like(self.nsel_tmp)
        self.out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)

    def local_scores(self, q) -> torch.Tensor:
        sh = self.sh
        csa.score_select(self.dl, q, sh.meta, sh.page_table, sh.seq_lens, self.Pr, self.Wr, 0,
                         self.sel_tmp, self.nsel_tmp, self.ws_local, scores_out=self.scores)
        return self.scores

    def attend(self, q, all_scores: List[torch.Tensor]):
        csa.select_scores(self.dg, torch.cat(all_scores, dim=2), self.sl_global, self.P, self.W,
                          self.budget, self.sel, self.n_sel, self.ws_global)
        csa.shard_selection(self.dg, self.sel, self.n_sel, self.lo, self.hi, self.sel_local,
                            self.n_local)
        sh = self.sh
        csa.decode(self.dl, q, sh.k_cache, sh.v_cache, sh.page_table, sh.seq_lens,
                   self.sel_local, self.n_local, self.Pr, self.Wr, self.out, self.ws_local,
                   lse=self.lse, scale=self.scale)
        return self.out, self.lse

    def merge(self, outs: List[torch.Tensor], lses: List[torch.Tensor]):
        out = torch.empty_like(outs[0])
        lse = torch.empty_like(lses[0])
        csa.merge_attention(torch.stack(outs), torch.stack(lses), out, lse)
        return out, lse


def gather_scores(exchange, plan: ShardPlan, s: torch.Tensor) -> List[torch.Tensor]:
    """All-gather of the ranks' score arrays [B][Hkv][p_{r+1} - p_r]: padded
    to the widest shard for the collective, trimmed after it."""
    sizes = [plan.hi(r) - plan.lo(r) for r in range(plan.world)]
    width = max(sizes)
    if s.shape[2] < width:
        pad = s.new_full(s.shape[:2] + (width - s.shape[2],), float("nan"))
        s = torch.cat([s, pad], dim=2)
    return [g[:, :, :n] for g, n in zip(exchange.all_gather(s), sizes)]


def cp_step(ops, exchange, q):
    """One rank's decode step: local scores, exchange, global selection and
    local attention, exchange, merge.  Returns (out, lse), the same on every
    rank; the global selection stays in (ops.sel, ops.n_sel)."""
    s = ops.local_scores(q)
    out_r, lse_r = ops.attend(q, gather_scores(exchange, ops.plan, s))
    outs = exchange.all_gather(out_r)
    lses = exchange.all_gather(lse_r)
    return ops.merge(outs, lses)


def shard_from_global(plan: ShardPlan, r: int, k_cache, v_cache, meta, page_table,
                      seq_lens: Sequence[int]) -> Shard:
    """Rank r's shard viewed inside a cache that holds every page (one-GPU
    emulation and tests): the page table's columns [p_r, p_{r+1})."""
    pt = page_table[:, plan.lo(r):plan.hi(r)].clone()       # own (aligned) storage
    sl = torch.tensor(plan.local_seq_lens(seq_lens, r), dtype=torch.int32,
                      device=page_table.device)
    return Shard(r, k_cache, v_cache, meta, pt, sl)
