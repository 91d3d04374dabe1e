#!/usr/bin/env python
"""Benchmark: combined sparse decode attention, tokens/s per layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ctx256k|ctx64k]

One step = one decode step of the whole hot path for every layer of the
workload: append the new token + metadata update (csa_meta_update), then
Quest scoring, top-k selection and the split-K sparse decode + merge in one
csa_sparse_attention call.  The default workload is the
12-layer, batch-4, 262144-token stack (32 query / 4 kv heads, head dim 128,
prefix 128, per-layer (window, budget) cycling through (512, 1024) ...
(4096, 8192)); its inputs are synthetic (seeded Gaussian q/K/V in a paged
cache with a random page permutation).  Each step is one CUDA graph of the
24 library calls; the K timed steps are replayed back to back between CUDA
events.  Every layer touches 150-235 MB (1.8-2.8 GB per step), more than the
126 MB L2, so no flush is needed between steps.

value = tokens/s per layer = B * layers * K / t (whole job: summed over
ranks, t = max over ranks).  ``roofline`` is measured on the dominant call
(scoring + selection at 256k) from graph replays over all 12 layers.
``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from dataclasses import replace

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from long_context_decoding_b200 import cost  # noqa: E402
from long_context_decoding_b200 import workloads as wl  # noqa: E402

METRIC = "decode attention tokens/s per layer at 64k/256k ctx, batch 4; % of HBM roofline"
UNIT = "tokens/s/layer"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("ctx256k", "ctx64k"), default="ctx256k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the 64k single-layer line")
    ap.add_argument("--profile", action="store_true",
                    help="timed steps only (for an ncu launch list): no baseline, e2e, clocks")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--layers", type=int, default=0,
                    help="use only the first N layers (small cases for ncu captures)")
    ap.add_argument("--layer-cfg", type=int, default=-1,
                    help="with --layers, start the stack's (window, budget) cycle at pair i "
                         "(e.g. --layers 1 --layer-cfg 3: one layer with the largest pair)")
    ap.add_argument("--no-fp8", action="store_true", help="skip the fp8-metadata line")
    ap.add_argument("--fp8-step", action="store_true",
                    help="with --profile: the timed steps score from the fp8 metadata copy "
                         "(csa_meta_update_fp8 + csa_sparse_attention_fp8), for ncu captures")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the compact sparse-vs-dense sweep of the default run")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the step: sparse (one call) vs dense decode over uniform "
                         "lengths 4k..256k and budgets 0/1024/4096/all, with a byte-based "
                         "cost-model fit; prints one JSON line")
    return ap.parse_args()


# ---------------------------------------------------------------- plumbing
class Dist:
    """One process per GPU (torchrun's RANK/LOCAL_RANK/WORLD_SIZE); the only
    collectives are the timing barrier and the max over ranks."""

    def __init__(self, backend: str | None = None, timeout_s: float = 180.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.backend = None
        if self.world > 1:
            import torch.distributed as dist
            backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.pg = dist
            self.backend = backend

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        dev = torch.device("cuda", self.local) if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def rank_workload(base: wl.Workload, rank: int, total_steps: int) -> wl.Workload:
    """The replica a rank decodes: the same shapes as `base`, its own seed.
    Ranks share nothing, so the path needs no collective (weak scaling)."""
    return replace(base, steps=total_steps, seed=base.seed + 1000 * rank)


def job_value(world: int, units_per_rank: int, t_max: float) -> float:
    """Whole-job throughput: units every rank processed over the slowest
    rank's device time."""
    return world * units_per_rank / t_max


def score_traffic():
    """DRAM bytes per launch of the scoring kernel from the committed ncu
    summary, or None when score.cu changed since those counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic_score_kernel.txt")) as f:
            rec = json.load(f)["score_kernel"]
        with open(os.path.join(ROOT, "long_context_decoding_b200", "csrc", "score.cu"), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
                return None, None
        return rec["dram_bytes_per_launch"], rec["workload"]
    except Exception:
        return None, None


def step_dram_traffic():
    """DRAM bytes per 256k layer step (all kernels of one append +
    csa_sparse_attention) from the committed ncu launch summary, or None
    when a kernel source changed since those counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic_layer_step.txt")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for name in sorted(rec["sources"]):
            with open(os.path.join(ROOT, "long_context_decoding_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["sources_sha256"]:
            return None
        return {"bytes_per_layer_step": rec["dram_bytes_per_layer_step"],
                "source": rec["source"]}
    except Exception:
        return None


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    Q = ("index,clocks.sm,clocks.max.sm,utilization.gpu,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        sel = []
        try:   # nvidia-smi numbers GPUs physically; select ours by UUID
            sel = ["-i", "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)]
        except Exception:
            pass
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100", *sel],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        text = self.f.read()
        os.unlink(self.f.name)
        return clocks_summary(text)


def clocks_summary(text: str):
    """Median SM clock, the maximum clock and the throttle reasons seen, from
    nvidia-smi CSV rows in the order of Clocks.Q (no header, no units); rows
    with the GPU at least 50% busy only, when there are any."""
    rows = [r.split(", ") for r in text.strip().splitlines() if r.count(",") >= 9]
    if not rows:
        return None
    busy = [r for r in rows if r[3].strip().isdigit() and int(r[3]) >= 50] or rows
    mhz = [float(r[1]) for r in busy if r[1].strip().replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in busy for i in range(4) if r[6 + i].strip() == "Active"})
    return {"sm_mhz": statistics.median(mhz) if mhz else None,
            "sm_max_mhz": float(busy[0][2]) if busy[0][2].strip().isdigit() else None,
            "reasons": reasons, "samples": len(busy)}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w: wl.Workload, seconds: float, steps: int = 0, warmup: int = 0,
                  threads: int = 0, dense: bool = False):
    """Time the CPU oracle on a bounded sample of workload ``w``: one
    sequence (all its kv-heads and query heads) of the first layer, full
    length, one decode step (scores -> top-k -> attention; with dense, the
    attention over every token) per iteration, on `threads` host threads (0:
    every core the process may use).
    Returns (tokens/s per layer, iterations, seconds, threads, sample)."""
    import oracle
    threads = oracle.set_threads(threads if threads > 0 else len(os.sched_getaffinity(0)))
    ws = replace(w, B=1, seq_lens=w.seq_lens[:1], layers=1, steps=0, spare_pages=0)
    c = wl.make_case(ws, "cpu", poison=False)
    window, budget = w.layer_window_budget(0)
    d = oracle.Dims(1, ws.Hq, ws.Hkv, ws.D, 16, ws.max_pages, ws.num_pages)
    h = dict(q=wl.bits(c.q), k=wl.bits(c.k_cache), v=wl.bits(c.v_cache),
             pt=c.page_table.numpy(), sl=c.seq_lens.numpy())
    scale = 1.0 / math.sqrt(ws.D)

    def one():
        if dense:
            oracle.attend(d, h["q"], h["k"], h["v"], h["pt"], h["sl"], 0, 0, None, None, 1,
                          scale, dense=True)
        else:
            oracle.step(d, h["q"], h["k"], h["v"], h["pt"], h["sl"], ws.prefix, window, budget,
                        max(1, budget // 16), scale)

    for _ in range(warmup):
        one()
    n, t0 = 0, time.perf_counter()
    while True:
        one()
        n += 1
        el = time.perf_counter() - t0
        if (steps and n >= steps) or (not steps and el >= seconds):
            break
    what = "dense attention" if dense else "decode step"
    return n / el, n, el, threads, (f"1 of {w.B} sequences of layer 0 (window {window}, budget "
                                    f"{budget}) at {w.seq_lens[0]} tokens, all {w.Hkv} kv-heads "
                                    f"and {w.Hq} query heads; one oracle {what} per "
                                    f"iteration, {n} iterations in {el:.1f} s")


def run_reference(args, dist: Dist, w: wl.Workload):
    if dist.rank != 0:
        return
    rate, n, el, threads, sample = oracle_sample(w, 0, steps=args.steps, warmup=args.warmup)
    line = {"metric": METRIC, "value": rate, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * el / n, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "layers": w.layers, "batch": w.B,
                       "ctx": w.seq_lens[0], "step": "one sequence, layer 0 (bounded sample)"},
            "cpu_baseline": {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU stack
class Stack:
    """All layers of a workload on one GPU, with per-step inputs resident."""

    def __init__(self, w: wl.Workload, dev):
        from long_context_decoding_b200 import csa
        self.csa = csa
        self.w = w
        self.dev = dev
        self.d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
        self.ws = csa.new_workspace(self.d, dev)
        self.layers = []
        for i in range(w.layers):
            c = wl.make_case(w, dev, layer=i)
            lay = csa.Layer(self.d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix,
                            c.window, c.budget, ws=self.ws)
            lay.rebuild_meta()
            lay.case = c
            self.layers.append(lay)
        L0 = torch.tensor(w.seq_lens, dtype=torch.int32, device=dev)
        self.lens = [(L0 + s + 1).contiguous() for s in range(w.steps)]
        self.inputs = [[wl.step_tokens(lay.case, s) for lay in self.layers]
                       for s in range(w.steps)]
        torch.cuda.synchronize()
        assert csa.device_status(self.ws) == 0

    def calls(self, s: int, q=None, nk=None, nv=None, what="all", layers=None):
        csa = self.csa
        for li in (layers if layers is not None else range(len(self.layers))):
            lay = self.layers[li]
            q_, nk_, nv_ = self.inputs[s][li]
            q_ = q[li] if q is not None else q_
            nk_ = nk[li] if nk is not None else nk_
            nv_ = nv[li] if nv is not None else nv_
            lens = self.lens[s]
            if what in ("all",):
                csa.meta_update(self.d, lay.k_cache, lay.v_cache, lay.meta, lay.page_table, lens,
                                nk_, nv_, 1, self.ws)
            if what in ("all", "sparse"):
                csa.sparse_attention(self.d, q_, lay.k_cache, lay.v_cache, lay.meta,
                                     lay.page_table, lens, lay.prefix, lay.window, lay.budget,
                                     lay.sel, lay.n_sel, lay.out, self.ws, lay.lse)
            if what in ("all_fp8",):
                csa.meta_update_fp8(self.d, lay.k_cache, lay.v_cache, lay.meta, lay.meta8,
                                    lay.page_table, lens, nk_, nv_, 1, self.ws)
                csa.sparse_attention_fp8(self.d, q_, lay.k_cache, lay.v_cache, lay.meta8,
                                         lay.page_table, lens, lay.prefix, lay.window,
                                         lay.budget, lay.sel, lay.n_sel, lay.out, self.ws,
                                         lay.lse)
            if what in ("select",):
                csa.score_select(self.d, q_, lay.meta, lay.page_table, lens, lay.prefix,
                                 lay.window, lay.budget, lay.sel, lay.n_sel, self.ws)
            if what in ("decode",):
                csa.decode(self.d, q_, lay.k_cache, lay.v_cache, lay.page_table, lens, lay.sel,
                           lay.n_sel, lay.prefix, lay.window, lay.out, self.ws, lay.lse)

    def launches_per_step(self) -> int:
        """Kernels of one step: per layer the metadata update, then the scoring
        kernel, the fused selection + decode kernel and the split-K combine
        when the one-call path applies (1 <= k < candidates, at most 32 units,
        at most 16384 candidates per unit), else scoring (when k chooses),
        selection, decode and combine."""
        w = self.w
        n = 0
        for lay in self.layers:
            k = lay.budget // 16
            n_max = w.max_pages - lay.prefix // 16 - lay.window // 16
            if 0 < k < n_max and n_max <= 16384 and w.B * w.Hkv <= 32:
                n += 1 + 3
            else:   # selection (or the full list), decode, combine; scores when k chooses
                n += 1 + (1 if 0 < k < n_max else 0) + 3
        return n

    def graph(self, fn):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                fn()
        torch.cuda.current_stream().wait_stream(s)
        return g

    def bytes_per_layer(self, s: int):
        """Algorithmic bytes of each layer at step s."""
        L = [x + s + 1 for x in self.w.seq_lens]
        return [cost.layer_bytes(L, self.w.Hq, self.w.Hkv, self.w.D, lay.prefix, lay.window,
                                 lay.budget) for lay in self.layers]


def time_graphs(graphs, reps=1):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        for g in graphs:
            g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 1000.0


def run_ours(args, dist: Dist, base: wl.Workload):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the CUDA path has no CPU fallback)")
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    K, W = args.steps, args.warmup
    st = Stack(rank_workload(base, dist.rank, K + W), dev)
    w = st.w
    nl = len(st.layers)
    what = "all"
    if args.fp8_step:
        if not args.profile:
            raise SystemExit("bench.py: --fp8-step is a profiling mode (use it with --profile)")
        for lay in st.layers:
            lay.meta8 = st.csa.new_meta8(st.d, st.dev)
            st.csa.meta_update_fp8(st.d, lay.k_cache, lay.v_cache, lay.meta, lay.meta8,
                                   lay.page_table, st.lens[0], None, None,
                                   st.d.max_pages_per_seq * 16, st.ws)
        what = "all_fp8"
    # eager pass over every step: sets kernel attributes, checks the flags
    for s in range(K + W):
        st.calls(s, what=what)
    torch.cuda.synchronize()
    assert st.csa.device_status(st.ws) == 0, "device flag after the eager pass"
    graphs = [st.graph(lambda s=s: st.calls(s, what=what)) for s in range(K + W)]
    for s in range(W):
        graphs[s].replay()
    clocks = None if args.profile else Clocks(dev)
    if clocks:   # ~1 s of untimed load so that the sampler sees the clock under load
        t_end = time.perf_counter() + 1.0
        while time.perf_counter() < t_end:
            for g in graphs[:W]:
                g.replay()
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    t = time_graphs(graphs[W:W + K])
    dist.barrier()
    clk = clocks.stop() if clocks else None
    t = dist.max(t)
    flags = st.csa.device_status(st.ws)
    value = job_value(dist.world, w.B * nl * K, t)
    t_layer = t / (K * nl)

    # per-layer algorithmic bytes over the timed steps (averaged)
    per_layer = [st.bytes_per_layer(s) for s in range(W, W + K)]
    layer_sparse = statistics.mean(sum(x["sparse"] for x in bl) / nl for bl in per_layer)
    meta_b = statistics.mean(sum(x["meta"] for x in bl) / nl for bl in per_layer)
    kv_b = statistics.mean(sum(x["kv"] + x["q_out"] for x in bl) / nl for bl in per_layer)
    peak, peak_kind = hbm_peak()

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world, "steps": K,
            "warmup": W, "ms_per_step": 1000 * t / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian q/K/V, random page permutation)",
            "config": {"workload": w.name, "layers": nl, "batch": w.B, "ctx": w.seq_lens[0],
                       "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D,
                       "prefix": w.prefix,
                       "window_budget": [[lay.window, lay.budget] for lay in st.layers],
                       "l2": "no flush: every layer moves > 126 MB (L2); "
                             f"{layer_sparse * nl / 1e9:.2f} GB per step",
                       "timing": "one CUDA graph per decode step, K graphs replayed between "
                                 "CUDA events; max over ranks"},
            "gpu_launches": st.launches_per_step() * K,
            "layer_step": {"us": 1e6 * t_layer, "algorithmic_bytes": layer_sparse,
                           "achieved_gbs": layer_sparse / t_layer / 1e9,
                           "frac_of_measured_peak": layer_sparse / t_layer / 1e9 / peak,
                           "frac_of_8tbs_nominal": layer_sparse / t_layer / 1e9 / NOMINAL_HBM_GBS},
            "device_flags": flags}

    if not args.profile:
        # ---- per-call timing: graph replays over all layers (inputs >> L2).
        # "score" is csa_score_select with budget 0 and a scores_out buffer:
        # the scoring kernel over every candidate, followed by a selection
        # kernel that has nothing to select.
        s_last = W + K - 1
        g_spa = st.graph(lambda: st.calls(s_last, what="sparse"))
        g_sel = st.graph(lambda: st.calls(s_last, what="select"))
        g_dec = st.graph(lambda: st.calls(s_last, what="decode"))
        sc_buf = torch.empty((w.B, w.Hkv, w.max_pages), dtype=torch.float32, device=dev)

        def score_only():
            for lay in st.layers:
                st.csa.score_select(st.d, st.inputs[s_last][st.layers.index(lay)][0], lay.meta,
                                    lay.page_table, st.lens[s_last], lay.prefix, lay.window, 0,
                                    lay.sel, lay.n_sel, st.ws, scores_out=sc_buf)

        g_sco = st.graph(score_only)
        reps = 5
        times = {}
        for name, g in (("score", g_sco), ("sparse_attention", g_spa), ("score_select", g_sel),
                        ("decode", g_dec)):
            time_graphs([g])
            times[name] = time_graphs([g], reps) / (reps * nl)
        bl = st.bytes_per_layer(s_last)
        meta_bytes = sum(x["meta"] for x in bl) / nl
        dec_bytes = sum(x["kv"] + x["q_out"] for x in bl) / nl
        calls = {"score": {"us": 1e6 * times["score"], "bytes": meta_bytes,
                           "gbs": meta_bytes / times["score"] / 1e9},
                 "sparse_attention": {"us": 1e6 * times["sparse_attention"],
                                      "bytes": meta_bytes + dec_bytes,
                                      "gbs": (meta_bytes + dec_bytes) / times["sparse_attention"]
                                      / 1e9},
                 "score_select": {"us": 1e6 * times["score_select"], "bytes": meta_bytes,
                                  "gbs": meta_bytes / times["score_select"] / 1e9},
                 "decode": {"us": 1e6 * times["decode"], "bytes": dec_bytes,
                            "gbs": dec_bytes / times["decode"] / 1e9}}
        ach = calls["score"]["gbs"]
        traffic, traffic_src = score_traffic()
        step_ach = layer_sparse / t_layer / 1e9
        step_traffic = step_dram_traffic()
        line["roofline"] = {
            "bound": "hbm", "scope": "layer step",
            "achieved": step_ach, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": step_ach / peak, "frac_of_8tbs_nominal": step_ach / NOMINAL_HBM_GBS,
            "traffic": step_traffic["bytes_per_layer_step"] if step_traffic else None,
            "traffic_source": step_traffic["source"] if step_traffic else None,
            "note": "achieved = algorithmic bytes of a layer step (metadata of the candidate "
                    "pages + K/V of the attended tokens + q/out; mean over the 12 layers and "
                    "the timed steps) / device time of a layer step (append + "
                    "csa_sparse_attention: scoring, selection, attention, combine) from the "
                    "timed graph replays",
            "kernel": "score_direct_kernel (Quest scoring; the largest share of the launch list)",
            "kernel_achieved": ach, "kernel_frac": ach / peak, "kernel_traffic": traffic,
            "kernel_traffic_source": (f"ncu dram__bytes_read+write per launch, {traffic_src}, "
                                      "profiles/traffic_layer_step_ctx256k.md")
                                     if traffic else None,
            "kernel_note": "metadata bytes of the candidate pages (|C| x 4D per unit) / "
                           "CUDA-event time per call, from graph replays of budget-0 "
                           "csa_score_select calls over the 12 layers (scoring kernel + an "
                           "empty selection launch)"}
        line["calls"] = calls
        line["clocks"] = clk

        # ---- the optional fp8 metadata copy on the same stack
        if not args.no_fp8:
            line["fp8_metadata"] = fp8_step(st, K, W, sc_buf, s_last, peak, dist)

        # ---- end to end through the C ABI from pinned host buffers
        if not args.no_e2e:
            line["e2e"] = e2e(st, K, W, dist)

        # ---- 64k single layer (the other context of the metric)
        if not args.no_secondary and base.name == wl.CTX256K.name:
            line["ctx64k"] = secondary_64k(dev, dist)
            line["many_units"] = secondary_many_units(dev, dist, line)
            line["context_parallel"] = secondary_context_parallel(dev, dist)

        # ---- sparse against dense over context length, and the cost model
        if not args.no_sweep and base.name == wl.CTX256K.name:
            line["sweep"] = compact_sweep(dev, dist)

        # ---- CPU oracle on a bounded sample
        if not args.no_cpu_baseline and dist.rank == 0 and dist.world == 1:
            rate, n, el, threads, sample = oracle_sample(base, args.cpu_seconds)
            r1, _, _, _, s1 = oracle_sample(base, args.cpu_seconds / 3, threads=1)
            rd, _, _, td, sd = oracle_sample(base, args.cpu_seconds / 3, dense=True)
            line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads,
                                    "kind": "oracle", "sample": sample,
                                    "one_core": {"value": r1, "cores": 1, "sample": s1},
                                    "dense": {"value": rd, "cores": td, "sample": sd}}
            if not args.no_secondary and base.name == wl.CTX256K.name:
                rec = oracle_planted_recall(dev)
                line["cpu_baseline"]["planted_recall_oracle"] = {
                    "workload": wl.CTX64K.name, "mean": rec["mean"], "min": rec["min"],
                    "per_unit": rec["per_unit"],
                    "note": "the oracle's top-k on the same seeded 64k inputs: the fraction of "
                            "the 32 planted pages per (sequence, kv-head) it selects"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def e2e(st: Stack, K: int, W: int, dist: Dist):
    """Per step: one H2D copy of the step's inputs (every layer's q, new_k
    and new_v, packed in one pinned host buffer), the 24 library calls on
    views of the device copy, and one D2H copy of every layer's output
    (the layers write into one device buffer); one CUDA graph per step, K
    steps timed."""
    nl = len(st.layers)
    shapes = [[t.shape for t in st.inputs[0][li]] for li in range(nl)]
    sizes = [[t.numel() for t in st.inputs[0][li]] for li in range(nl)]
    per_step = sum(sum(x) for x in sizes)
    dev = st.dev
    dev_in = torch.empty(per_step, dtype=torch.bfloat16, device=dev)
    views, at = [], 0
    for li in range(nl):
        v = []
        for shp, n in zip(shapes[li], sizes[li]):
            v.append(dev_in[at:at + n].view(shp))
            at += n
        views.append(v)
    host_in = []
    for s in range(K + W):
        h = torch.cat([t.reshape(-1).cpu() for li in range(nl) for t in st.inputs[s][li]])
        host_in.append(h.pin_memory())
    out_all = torch.empty((nl,) + tuple(st.layers[0].out.shape), dtype=torch.bfloat16, device=dev)
    saved = [lay.out for lay in st.layers]
    for li, lay in enumerate(st.layers):
        lay.out = out_all[li]
    host_out = [torch.empty(out_all.shape, dtype=torch.bfloat16).pin_memory()
                for _ in range(K + W)]

    def step(s):
        dev_in.copy_(host_in[s], non_blocking=True)
        st.calls(s, q=[v[0] for v in views], nk=[v[1] for v in views],
                 nv=[v[2] for v in views])
        host_out[s].copy_(out_all, non_blocking=True)

    graphs = [st.graph(lambda s=s: step(s)) for s in range(K + W)]
    for s in range(W):
        graphs[s].replay()
    torch.cuda.synchronize()
    dist.barrier()
    t = dist.max(time_graphs(graphs[W:W + K]))
    del graphs
    for lay, o in zip(st.layers, saved):
        lay.out = o
    h2d = host_in[0].numel() * host_in[0].element_size()
    d2h = host_out[0].numel() * host_out[0].element_size()
    return {"value": dist.world * st.w.B * nl * K / t, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "path": "one pinned host -> device copy of the step's inputs (all layers' q, new "
                    "K, new V), csa_meta_update / csa_sparse_attention per layer, one device -> "
                    "pinned host copy of all layers' outputs; one CUDA graph per step"}


def fp8_step(st: Stack, K: int, W: int, sc_buf, s_last: int, peak: float, dist: Dist):
    """The same 12-layer steps with the scores read from the fp8 metadata copy
    (csa_meta_update_fp8 + csa_sparse_attention_fp8 per layer): an option with
    a looser Quest bound (the selection can differ from the bf16 one), not the
    headline."""
    csa = st.csa
    w = st.w
    for lay in st.layers:
        lay.meta8 = csa.new_meta8(st.d, st.dev)
        csa.meta_update_fp8(st.d, lay.k_cache, lay.v_cache, lay.meta, lay.meta8, lay.page_table,
                            st.lens[0], None, None, st.d.max_pages_per_seq * 16, st.ws)
    for s in range(K + W):
        st.calls(s, what="all_fp8")
    torch.cuda.synchronize()
    graphs = [st.graph(lambda s=s: st.calls(s, what="all_fp8")) for s in range(K + W)]
    for s in range(W):
        graphs[s].replay()
    torch.cuda.synchronize()
    dist.barrier()
    t = dist.max(time_graphs(graphs[W:W + K]))
    nl = len(st.layers)

    def score_only():
        for li, lay in enumerate(st.layers):
            csa.score_select_fp8(st.d, st.inputs[s_last][li][0], lay.meta8, lay.page_table,
                                 st.lens[s_last], lay.prefix, lay.window, 0, lay.sel, lay.n_sel,
                                 st.ws, scores_out=sc_buf)

    g = st.graph(score_only)
    time_graphs([g])
    ts = time_graphs([g], 5) / (5 * nl)
    bl = st.bytes_per_layer(s_last)
    cand = sum(x["meta"] for x in bl) / nl / (4 * w.D)          # candidate rows per layer
    meta8_bytes = cand * (2 * w.D + 16)
    for lay in st.layers:
        lay.meta8 = None
    torch.cuda.empty_cache()
    return {"value": dist.world * w.B * nl * K / t, "unit": UNIT, "ms_per_step": 1000 * t / K,
            "layer_step_us": 1e6 * t / (K * nl),
            "score_call": {"us": 1e6 * ts, "bytes": meta8_bytes,
                           "gbs": meta8_bytes / ts / 1e9,
                           "frac_of_measured_peak": meta8_bytes / ts / 1e9 / peak},
            "note": "scores from the E4M3 metadata copy (min rounded down, max up, per-row "
                    "power-of-two scale; 2D + 16 bytes per row instead of 4D); a looser "
                    "upper bound, so the selection can differ from the bf16 one"}


def secondary_64k(dev, dist: Dist):
    """The 64k single-layer workload: one layer step (one
    csa_sparse_attention call: score, select, decode; no append) per graph;
    a 256 MB read before every replay flushes L2 (the layer itself moves only
    ~84 MB), and batches of replays are timed (graph_time).  The flush reads
    rather than writes, so that no dirty L2 lines are written back during the
    timed replay."""
    from long_context_decoding_b200 import csa
    w = wl.CTX64K
    c = wl.make_case(w, dev)
    d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
    lay = csa.Layer(d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix, w.window,
                    w.budget)
    lay.rebuild_meta()
    scrub = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MB
    sink = torch.zeros((), device=dev)

    def flush():
        torch.sum(scrub, dim=0, out=sink)

    t = dist.max(graph_time(lambda: lay.step(c.q, fused=True), 20, 5, flush))
    by = cost.layer_bytes(w.seq_lens, w.Hq, w.Hkv, w.D, w.prefix, w.window, w.budget)
    peak, _ = hbm_peak()
    ach = by["sparse"] / t / 1e9
    # dense comparison on the same cache
    out = torch.empty_like(lay.out)
    tdn = graph_time(lambda: csa.decode_full(d, c.q, c.k_cache, c.v_cache, c.page_table,
                                             c.seq_lens, out, lay.ws), 10, 3, flush)
    lay.step(c.q, fused=True)
    recall = planted_recall(lay.sel.cpu().numpy(), lay.n_sel.cpu().numpy(),
                            c.planted_pages.cpu().numpy())
    return {"workload": w.name, "value": dist.world * w.B / t, "unit": UNIT,
            "us_per_layer_step": 1e6 * t, "algorithmic_bytes": by["sparse"],
            "frac": ach / peak,
            "planted_recall": {"mean": recall["mean"], "min": recall["min"],
                               "per_unit": recall["per_unit"],
                               "note": "fraction of the 32 q-aligned planted pages per "
                                       "(sequence, kv-head) that the one-call selection holds "
                                       "(a measurement; the oracle's own figure is in "
                                       "cpu_baseline.planted_recall_oracle)"},
            "achieved_gbs": ach, "frac_of_measured_peak": ach / peak,
            "frac_of_8tbs_nominal": ach / NOMINAL_HBM_GBS,
            "dense_us": 1e6 * tdn, "dense_gbs": by["dense"] / tdn / 1e9,
            "speedup_vs_dense": tdn / t,
            "timing": "batches of 20 graph replays, each after a 256 MB L2 flush (read); the flush time subtracted; median of 3 batches"}


def secondary_many_units(dev, dist: Dist, line):
    """One layer step of the 64k decode at batch 8 x 8 kv-heads (64
    (sequence, kv-head) units, D = 128): one csa_sparse_attention call,
    which beyond 32 units runs as scoring, selection, decode and combine
    launches.  Timed like the 64k line (L2 read-flush before every replay);
    its per-byte rate is set against the 8-unit 64k layer and the 256k
    stack's layer step."""
    from long_context_decoding_b200 import csa
    w = wl.CTX64K_B8
    c = wl.make_case(w, dev)
    d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
    lay = csa.Layer(d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix, w.window,
                    w.budget)
    lay.rebuild_meta()
    scrub = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MB
    sink = torch.zeros((), device=dev)

    def flush():
        torch.sum(scrub, dim=0, out=sink)

    t = dist.max(graph_time(lambda: lay.step(c.q, fused=True), 20, 5, flush))
    flags = csa.device_status(lay.ws)
    by = cost.layer_bytes(w.seq_lens, w.Hq, w.Hkv, w.D, w.prefix, w.window, w.budget)
    peak, _ = hbm_peak()
    ach = by["sparse"] / t / 1e9
    ref64 = line.get("ctx64k", {}).get("achieved_gbs")
    ref256 = line.get("layer_step", {}).get("achieved_gbs")
    del lay, c
    torch.cuda.empty_cache()
    return {"workload": w.name, "units": w.B * w.Hkv, "value": dist.world * w.B / t,
            "unit": UNIT, "us_per_layer_step": 1e6 * t, "algorithmic_bytes": by["sparse"],
            "achieved_gbs": ach, "frac_of_measured_peak": ach / peak,
            "rate_vs_ctx64k": ach / ref64 if ref64 else None,
            "rate_vs_256k_layer_step": ach / ref256 if ref256 else None,
            "device_flags": flags,
            "path": "more than 32 units: scoring, cluster selection, decode (prefix/window "
                    "pages during the selection) and combine as separate launches",
            "timing": "batches of 20 graph replays, each after a 256 MB L2 flush (read); the "
                      "flush time subtracted; median of 3 batches"}


PEER_GBS = 770.0   # measured NVLink peer-copy bandwidth per direction on this hardware


def secondary_context_parallel(dev, dist: Dist):
    """Context parallelism emulated on one GPU: the 256k stack's first layer
    (window 512, budget 1024) with every sequence's pages split over R = 2
    and 4 ranks.  Each rank's kernels are timed as graph replays after an L2
    flush, one rank after another: its local scoring, then its step after
    the score exchange (the global selection from the gathered scores, its
    share of the selection and its decode), then the merge after the partial
    exchange.  The two all-gathers are not run (one GPU): their bytes per
    rank are reported with the time they take at the measured peer
    bandwidth, as a bound, not a measurement."""
    from long_context_decoding_b200 import context_parallel as cp
    from long_context_decoding_b200 import csa
    w = replace(wl.CTX256K, layers=1)
    c = wl.make_case(w, dev, layer=0)
    d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_sel)
    lay = csa.Layer(d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix, c.window,
                    c.budget)
    lay.rebuild_meta()
    scrub = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MB
    sink = torch.zeros((), device=dev)

    def flush():
        torch.sum(scrub, dim=0, out=sink)

    t_one = dist.max(graph_time(lambda: lay.step(c.q, fused=True), 20, 5, flush))
    ref = lay.out.float().clone()
    lens = [int(x) for x in c.seq_lens.cpu()]
    res = {"workload": w.name + " layer 0", "single_gpu_us": 1e6 * t_one, "ranks": []}
    for R in (2, 4):
        plan = cp.plan_shards(w.max_pages, R, w.prefix, c.window, lens)
        ops = [cp.CudaOps(plan, d, cp.shard_from_global(plan, r, c.k_cache, c.v_cache, lay.meta,
                                                        c.page_table, lens),
                          c.seq_lens, w.prefix, c.window, c.budget) for r in range(R)]
        scores = [o.local_scores(c.q).clone() for o in ops]
        parts = [tuple(x.clone() for x in o.attend(c.q, scores)) for o in ops]
        out, _ = ops[0].merge([x[0] for x in parts], [x[1] for x in parts])
        torch.cuda.synchronize()
        err = float((out.float() - ref).abs().max())
        t_sc = [dist.max(graph_time(lambda o=o: o.local_scores(c.q), 10, 3, flush)) for o in ops]
        t_at = [dist.max(graph_time(lambda o=o: o.attend(c.q, scores), 10, 3, flush)) for o in ops]
        t_mg = dist.max(graph_time(lambda: ops[0].merge([x[0] for x in parts],
                                                        [x[1] for x in parts]), 10, 3, flush))
        score_bytes = [4 * w.B * w.Hkv * (plan.hi(r) - plan.lo(r)) for r in range(R)]
        part_bytes = w.B * w.Hq * (2 * w.D + 4)
        recv = max(sum(score_bytes) - sb for sb in score_bytes) + (R - 1) * part_bytes
        comp = max(a + b for a, b in zip(t_sc, t_at)) + t_mg
        res["ranks"].append({
            "R": R, "score_us": [1e6 * t for t in t_sc], "select_decode_us": [1e6 * t for t in t_at],
            "merge_us": 1e6 * t_mg, "rank_kernels_us_max": 1e6 * comp,
            "exchange_bytes_received_per_rank": recv,
            "exchange_us_at_peer_bandwidth": 1e6 * recv / (PEER_GBS * 1e9),
            "max_abs_diff_vs_single_gpu": err})
        del ops
        torch.cuda.empty_cache()
    res["note"] = ("ranks emulated one after another on one GPU; the all-gathers are not run: "
                   "exchange_us_at_peer_bandwidth is bytes / 770 GB/s, a bound")
    del lay, c
    torch.cuda.empty_cache()
    return res


def planted_recall(sel, nsel, planted):
    """Per (sequence, kv-head): the fraction of its planted pages that the
    selection sel[b][g][:nsel[b][g]] holds."""
    per = []
    for b in range(planted.shape[0]):
        for g in range(planted.shape[1]):
            got = set(int(x) for x in sel[b, g, :int(nsel[b, g])])
            want = [int(x) for x in planted[b, g]]
            per.append(sum(p in got for p in want) / len(want))
    return {"mean": sum(per) / len(per), "min": min(per), "per_unit": per}


def oracle_planted_recall(dev):
    """The oracle's selection on the 64k planted workload (same seeded
    inputs, copied to the host) and its planted-page recall."""
    import oracle
    w = wl.CTX64K
    c = wl.make_case(w, dev)
    d = oracle.Dims(w.B, w.Hq, w.Hkv, w.D, 16, w.max_pages, w.num_pages)
    q, k = wl.bits(c.q), wl.bits(c.k_cache)
    pt, sl = c.page_table.cpu().numpy(), c.seq_lens.cpu().numpy()
    planted = c.planted_pages.cpu().numpy()
    del c
    torch.cuda.empty_cache()
    oracle.set_threads(len(os.sched_getaffinity(0)))
    sc = oracle.scores(d, q, k, pt, sl, w.prefix, w.window)
    sel, nsel = oracle.select(d, sc, sl, w.prefix, w.window, w.budget, w.max_sel)
    return planted_recall(sel, nsel, planted)


def graph_time(fn, reps: int, warm: int, flush) -> float:
    """CUDA-event time (s) of one graph replay of fn with L2 flushed (by a
    read) before it: reps x (flush + replay) minus reps x flush, each between
    one pair of events (a single replay is too short for the event clock's
    2 us granularity on this system); the median of three such batches."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(warm):
        flush()
        g.replay()
    torch.cuda.synchronize()

    def batch(with_fn: bool) -> float:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            flush()
            if with_fn:
                g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / 1000.0

    return statistics.median((batch(True) - batch(False)) / reps for _ in range(3))


def sweep_points(dev, grid, budgets, reps: int, warm: int):
    """Sparse (csa_sparse_attention) against dense (csa_decode_full) decode on
    the same cache, batch 4, 16 query / 4 kv heads, D 128, prefix 128, window
    1024, at every length of `grid` and every budget of `budgets` (None: the
    whole context); each time from graph replays with L2 flushed (graph_time).
    Returns the points and the cost-model fits over them."""
    from long_context_decoding_b200 import csa
    scrub = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MB
    sink = torch.zeros((), device=dev)

    def flush():
        torch.sum(scrub, dim=0, out=sink)

    points = []
    for L in grid:
        w = replace(wl.SWEEP, name=f"b4_h16x4_d128_ctx{L}", seq_lens=(L,) * 4)
        c = wl.make_case(w, dev)
        d = csa.make_dims(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.num_pages, w.max_pages)
        lay = csa.Layer(d, c.k_cache, c.v_cache, c.page_table, c.seq_lens, w.prefix, w.window,
                        0)
        lay.rebuild_meta()
        out = torch.empty_like(lay.out)
        t_dense = graph_time(lambda: csa.decode_full(d, c.q, c.k_cache, c.v_cache,
                                                       c.page_table, c.seq_lens, out, lay.ws),
                               reps, warm, flush)
        for budget in budgets:
            lay.budget = PS_TOKENS * w.max_pages if budget is None else budget
            t = graph_time(lambda: lay.step(c.q, fused=True), reps, warm, flush)
            by = cost.layer_bytes(w.seq_lens, w.Hq, w.Hkv, w.D, w.prefix, w.window, budget)
            points.append({"L": L, "budget": "all" if budget is None else budget,
                           "path": cost.path_of(L, w.prefix, w.window, budget),
                           "sparse_us": 1e6 * t, "dense_us": 1e6 * t_dense,
                           "speedup": t_dense / t, "sparse_bytes": by["sparse"],
                           "dense_bytes": by["dense"], "sparse_gbs": by["sparse"] / t / 1e9})
        assert csa.device_status(lay.ws) == 0
        del c, lay, out
        torch.cuda.empty_cache()
    # one fixed cost for every point
    x = [p["sparse_bytes"] for p in points]
    y = [p["sparse_us"] * 1e-6 for p in points]
    n = len(x)
    mx, my = sum(x) / n, sum(y) / n
    slope = sum((a - mx) * (b - my) for a, b in zip(x, y)) / sum((a - mx) ** 2 for a in x)
    t0 = my - slope * mx
    for p in points:
        p["model_us"] = 1e6 * (t0 + slope * p["sparse_bytes"])
    worst = max(abs(p["model_us"] - p["sparse_us"]) / p["sparse_us"] for p in points)
    per_path = cost.fit_per_path(points)
    for p in points:
        p["model_per_path_us"] = (per_path["t0_us"][p["path"]]
                                  + p["sparse_bytes"] / (per_path["bw_gbs"] * 1e3))
    fits = {"cost_model": {"t0_us": 1e6 * t0, "bw_gbs": 1.0 / slope / 1e9, "max_rel_err": worst,
                           "form": "t = t0 + algorithmic bytes / bw"},
            "cost_model_per_path": per_path}
    return points, fits


def compact_sweep(dev, dist: Dist):
    """The sweep's key points for the default run: sparse against dense at
    16k, 32k, 64k and 256k for budgets 0, 1024 and 4096, with the per-path
    cost-model fit over them."""
    points, fits = sweep_points(dev, (16384, 32768, 65536, 262144), (0, 1024, 4096), 10, 3)
    keep = ("L", "budget", "path", "sparse_us", "dense_us", "speedup", "sparse_gbs",
            "model_per_path_us")
    return {"config": "batch 4, 16 query / 4 kv heads, D 128, prefix 128, window 1024, uniform "
                      "lengths; csa_sparse_attention against csa_decode_full on the same cache; "
                      "graph replays after a 256 MB L2 read-flush, median of 3 batches",
            "points": [{k: p[k] for k in keep} for p in points],
            "sparse_faster_than_dense_for_all_L_ge_32k":
                all(p["sparse_us"] < p["dense_us"] for p in points if p["L"] >= 32768),
            "cost_model_per_path": fits["cost_model_per_path"]}


def run_sweep(args, dist: Dist):
    """The full sweep (--sweep): every length of the grid, budgets 0, 1024,
    4096 and all; the cost model t = t0 + bytes / bw fitted by least squares,
    with one fixed cost and with one per path."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the CUDA path has no CPU fallback)")
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    points, fits = sweep_points(dev, wl.SWEEP_GRID, wl.SWEEP_BUDGETS, args.steps, args.warmup)
    # a budget of "all" attends to every token: the same work as dense
    beats = all(p["sparse_us"] < p["dense_us"] for p in points
                if p["L"] >= 32768 and p["budget"] != "all")
    all_ratio = min(p["dense_us"] / p["sparse_us"] for p in points if p["budget"] == "all")
    line = {"metric": "sparse vs dense decode layer step over context length and budget",
            "unit": "us", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "dtype": "bf16", "data": "synthetic (seeded Gaussian q/K/V, random page permutation)",
            "config": {"workload": wl.SWEEP.name + " (uniform lengths)", "batch": 4,
                       "q_heads": 16, "kv_heads": 4, "head_dim": 128, "prefix": 128,
                       "window": 1024, "l2": "256 MB read between replays",
                       "timing": "median of graph replays, CUDA events"},
            "points": points, **fits,
            "sparse_faster_than_dense_for_all_L_ge_32k": beats,
            "all_budget_min_speedup_vs_dense": all_ratio}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


PS_TOKENS = 16


def main():
    args = parse_args()
    dist = Dist()
    if args.sweep:
        try:
            run_sweep(args, dist)
        finally:
            dist.close()
        return
    base = wl.CTX256K if args.workload == "ctx256k" else replace(wl.CTX64K, steps=0)
    if args.layers:
        base = replace(base, layers=args.layers)
    if args.layer_cfg >= 0 and base.layer_cfgs:
        i = args.layer_cfg % len(base.layer_cfgs)
        base = replace(base, layer_cfgs=base.layer_cfgs[i:] + base.layer_cfgs[:i])
    try:
        if args.impl == "reference":
            run_reference(args, dist, base)
        else:
            run_ours(args, dist, base)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
