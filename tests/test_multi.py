"""Host logic of the N>1 benchmark path, as two `gloo` ranks on the CPU.

Several GPUs decode independent replicas (their own sequences; no data-path
collective).  What the ranks share is only the timing protocol: a barrier
on both sides of the timed region, the max of the device times over ranks,
and whole-job throughput = units of all ranks / that max.  The reference
arm runs on rank 0 alone.  These tests launch two processes (spawn) that run
exactly those pieces of bench.py.
"""
import contextlib
import io
import os
import socket
import sys
from argparse import Namespace

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from long_context_decoding_b200 import workloads as wl

    d = bench.Dist(backend="gloo", timeout_s=60)
    rec = {"rank": d.rank, "world": d.world}
    d.barrier()
    # device time of this rank's timed region: rank r is slower by r
    t = 0.25 + 0.5 * rank
    rec["t_max"] = d.max(t)
    steps = 3
    w = bench.rank_workload(wl.TINY, rank, steps)
    rec["seed"] = w.seed
    rec["steps"] = w.steps
    units = w.B * w.layers * steps
    rec["value"] = bench.job_value(d.world, units, rec["t_max"])
    rec["units"] = units
    c = wl.make_case(w, "cpu", poison=False)
    rec["q"] = c.q.float().clone()
    rec["k_shape"] = tuple(c.k_cache.shape)
    # reference arm: rank 0 prints the one line, the others print nothing
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(Namespace(steps=1, warmup=0, gpus=world), d, wl.TINY)
    rec["stdout"] = buf.getvalue()
    d.barrier()
    d.close()
    torch.save(rec, os.path.join(out_dir, f"rank{rank}.pt"))


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("multi"))
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    return [torch.load(os.path.join(out, f"rank{r}.pt"), weights_only=False) for r in (0, 1)]


def test_ranks_join_one_group(two_ranks):
    assert [r["rank"] for r in two_ranks] == [0, 1]
    assert all(r["world"] == 2 for r in two_ranks)


def test_time_is_max_over_ranks(two_ranks):
    assert all(r["t_max"] == pytest.approx(0.75) for r in two_ranks)


def test_job_value_counts_every_rank(two_ranks):
    r = two_ranks[0]
    assert r["value"] == pytest.approx(2 * r["units"] / 0.75)
    assert two_ranks[0]["value"] == two_ranks[1]["value"]


def test_replicas_differ_but_keep_shapes(two_ranks):
    a, b = two_ranks
    assert a["seed"] != b["seed"] and a["steps"] == b["steps"] == 3
    assert a["k_shape"] == b["k_shape"]
    assert a["q"].shape == b["q"].shape
    assert not torch.equal(a["q"], b["q"])


def test_reference_arm_prints_on_rank0_only(two_ranks):
    import json
    lines = [ln for ln in two_ranks[0]["stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert two_ranks[1]["stdout"] == ""
