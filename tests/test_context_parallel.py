"""Context parallelism on the CPU: the page split, and one decode step of
two and three `gloo` ranks whose four compute steps are done by the oracle
(scores, selection, attention) and by the log-sum-exp merge written out
here, against the oracle's single-process step.  What this checks is the
host logic of long_context_decoding_b200/context_parallel.py: which shard
each rank holds, its prefix and window, the order of the collectives and
what each rank contributes; the kernels themselves are checked on the GPU
(test_gpu_context_parallel.py)."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from long_context_decoding_b200 import context_parallel as cp
from long_context_decoding_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PS = 16


def lse_merge(outs, lses):
    """exp-weighted merge of normalised partial outputs (float64)."""
    lses = np.stack(lses)                       # [R][B][Hq]
    outs = np.stack(outs)                       # [R][B][Hq][D]
    M = lses.max(axis=0)
    safe = np.where(np.isfinite(M), M, 0.0)
    w = np.exp(lses - safe)                     # 0 for parts with lse = -inf
    tot = w.sum(axis=0)
    out = np.where(tot[..., None] > 0, (w[..., None] * outs).sum(axis=0) /
                   np.where(tot > 0, tot, 1.0)[..., None], 0.0)
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return out, lse


class OracleOps:
    """The steps of one rank, computed by the oracle on the host."""

    def __init__(self, plan, r, w, a, max_sel, scale):
        self.plan, self.r = plan, r
        self.lo, self.hi = plan.lo(r), plan.hi(r)
        self.a, self.w = a, w
        self.max_sel, self.scale = max_sel, scale
        self.Pr, self.Wr = plan.local_prefix_window(r, w.prefix, w.window)
        self.dl = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, self.hi - self.lo, w.num_pages)
        self.dg = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
        self.pt = np.ascontiguousarray(a["pt"][:, self.lo:self.hi])
        self.sl = np.array(plan.local_seq_lens(a["sl"], r), np.int32)

    def local_scores(self, q):
        a = self.a
        s = oracle.scores(self.dl, a["q"], a["k"], self.pt, self.sl, self.Pr, self.Wr)
        return torch.from_numpy(np.ascontiguousarray(s))

    def attend(self, q, all_scores):
        a, w = self.a, self.w
        g = torch.cat(all_scores, dim=2).numpy()
        self.sel, self.n_sel = oracle.select(self.dg, g, a["sl"], w.prefix, w.window, w.budget,
                                             self.max_sel)
        sel_l = np.full_like(self.sel, -1)
        n_l = np.zeros_like(self.n_sel)
        for b in range(w.B):
            for h in range(w.Hkv):
                p = self.sel[b, h, :self.n_sel[b, h]]
                p = p[(p >= self.lo) & (p < self.hi)] - self.lo
                sel_l[b, h, :len(p)] = p
                n_l[b, h] = len(p)
        out, lse = oracle.attend(self.dl, a["q"], a["k"], a["v"], self.pt, self.sl, self.Pr,
                                 self.Wr, sel_l, n_l, self.max_sel, self.scale)
        return torch.from_numpy(out), torch.from_numpy(lse)

    def merge(self, outs, lses):
        out, lse = lse_merge([o.numpy() for o in outs], [x.numpy() for x in lses])
        return torch.from_numpy(out), torch.from_numpy(lse)


def host_case(w):
    c = wl.make_case(w, "cpu")
    return {"q": wl.bits(c.q), "k": wl.bits(c.k_cache), "v": wl.bits(c.v_cache),
            "pt": c.page_table.numpy(), "sl": c.seq_lens.numpy()}


CP_SMALL = wl.Workload("cp_small", B=2, Hq=4, Hkv=2, D=32, seq_lens=(1500, 1203), prefix=40,
                       window=100, budget=160, seed=21)


def test_plan_splits_pages_evenly_and_checks_prefix_and_window():
    plan = cp.plan_shards(100, 3, 40, 100, (1500, 1203))
    assert plan.splits == (0, 33, 66, 100) and plan.world == 3
    assert plan.local_seq_lens((1500, 1203), 0) == [528, 528]
    assert plan.local_seq_lens((1500, 1203), 2) == [1500 - 1056, 1203 - 1056]
    assert plan.local_prefix_window(0, 40, 100) == (40, 0)
    assert plan.local_prefix_window(1, 40, 100) == (0, 0)
    assert plan.local_prefix_window(2, 40, 100) == (0, 100)
    with pytest.raises(ValueError):         # a window reaching into rank 1's pages
        cp.plan_shards(100, 3, 40, 300, (1500, 1203))
    with pytest.raises(ValueError):         # a prefix longer than rank 0's pages
        cp.plan_shards(100, 3, 600, 100, (1500, 1203))
    with pytest.raises(ValueError):         # a sequence that ends before the last rank
        cp.plan_shards(100, 3, 40, 100, (1500, 900))
    assert cp.plan_shards(7, 1, 10**6, 10**6, (100,)).splits == (0, 7)


def test_shards_partition_the_candidates():
    """The ranks' candidate pages (with their local prefix/window) are the
    global candidates, each on exactly one rank."""
    w, a = CP_SMALL, host_case(CP_SMALL)
    plan = cp.plan_shards(w.max_pages, 3, w.prefix, w.window, a["sl"])
    dg = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
    glob = oracle.scores(dg, a["q"], a["k"], a["pt"], a["sl"], w.prefix, w.window)
    parts = [OracleOps(plan, r, w, a, w.max_sel, 1.0).local_scores(None).numpy()
             for r in range(3)]
    cat = np.concatenate(parts, axis=2)
    np.testing.assert_array_equal(np.isnan(cat), np.isnan(glob))
    np.testing.assert_array_equal(cat[~np.isnan(cat)], glob[~np.isnan(glob)])


class ListExchange:
    """all_gather within one process, over the ranks' values of a phase."""

    def __init__(self, values):
        self.values = values

    def all_gather(self, t):
        return list(self.values)


def _worker(rank, world, port, out_dir):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, a = CP_SMALL, host_case(CP_SMALL)
    plan = cp.plan_shards(w.max_pages, world, w.prefix, w.window, a["sl"])
    ops = OracleOps(plan, rank, w, a, w.max_sel, 1.0 / math.sqrt(w.D))
    out, lse = cp.cp_step(ops, cp.TorchExchange(), None)
    torch.save({"out": out, "lse": lse, "sel": ops.sel, "n_sel": ops.n_sel},
               os.path.join(out_dir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_reproduce_the_single_process_step(world, tmp_path):
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    w, a = CP_SMALL, host_case(CP_SMALL)
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, PS, w.max_pages, w.num_pages)
    ref = oracle.step(od, a["q"], a["k"], a["v"], a["pt"], a["sl"], w.prefix, w.window,
                      w.budget, w.max_sel, 1.0 / math.sqrt(w.D))
    for r in range(world):
        got = torch.load(os.path.join(tmp_path, f"r{r}.pt"), weights_only=False)
        np.testing.assert_array_equal(got["n_sel"], ref["nsel"])
        for b in range(w.B):
            for h in range(w.Hkv):
                k = int(ref["nsel"][b, h])
                np.testing.assert_array_equal(got["sel"][b, h, :k], ref["sel"][b, h, :k])
        np.testing.assert_allclose(got["out"].numpy(), ref["out"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got["lse"].numpy(), ref["lse"], rtol=0, atol=1e-12)


def test_lse_merge_of_two_halves_is_the_whole_softmax():
    """The merge itself, against a softmax written out on random logits."""
    rng = np.random.default_rng(0)
    s = rng.normal(size=(3, 50)) * 4
    v = rng.normal(size=(50, 8))
    def attn(idx):
        z = s[:, idx]
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        return (p @ v[idx]) / p.sum(axis=1, keepdims=True), m[:, 0] + np.log(p.sum(axis=1))
    whole = attn(np.arange(50))
    parts = [attn(np.arange(0, 20)), attn(np.arange(20, 50))]
    out, lse = lse_merge([p[0][None] for p in parts], [p[1][None] for p in parts])
    np.testing.assert_allclose(out[0], whole[0], atol=1e-12)
    np.testing.assert_allclose(lse[0], whole[1], atol=1e-12)
    # a part with nothing attended contributes nothing
    empty = (np.zeros((3, 8)), np.full(3, -np.inf))
    out2, lse2 = lse_merge([parts[0][0][None], empty[0][None]],
                           [parts[0][1][None], empty[1][None]])
    np.testing.assert_allclose(out2[0], parts[0][0], atol=1e-12)
    np.testing.assert_allclose(lse2[0], parts[0][1], atol=1e-12)
