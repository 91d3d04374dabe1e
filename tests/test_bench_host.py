"""Host-side logic of bench.py that needs no GPU: the clock summary from
nvidia-smi rows, the DRAM-traffic records keyed to the kernel sources, and
the planted-page recall."""
import json
import os
import shutil

import numpy as np

import bench


def _row(util, mhz, active="Not Active", hw="Not Active", power_cap="Not Active"):
    # index, clocks.sm, clocks.max.sm, utilization.gpu, power.draw, reasons.active,
    # hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    return f"0, {mhz}, 1965, {util}, 700.5, {active}, {hw}, Not Active, Not Active, {power_cap}"


def test_clocks_summary_uses_busy_rows_and_collects_reasons():
    text = "\n".join([_row(0, 345), _row(0, 345), _row(97, 1965), _row(99, 1950),
                      _row(98, 1965, power_cap="Active"), "garbage line"])
    s = bench.clocks_summary(text)
    assert s["samples"] == 3                    # the idle rows are left out
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clocks_summary_without_busy_rows_or_rows():
    s = bench.clocks_summary("\n".join([_row(10, 1200, hw="Active"), _row(20, 1300)]))
    assert s["samples"] == 2 and s["sm_mhz"] == 1250.0 and s["reasons"] == ["hw_slowdown"]
    assert bench.clocks_summary("") is None


def _copy_tree(tmp_path):
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(bench.ROOT, "profiles"), root / "profiles")
    shutil.copytree(os.path.join(bench.ROOT, "long_context_decoding_b200", "csrc"),
                    root / "long_context_decoding_b200" / "csrc")
    return root


def test_traffic_records_follow_their_sources(tmp_path, monkeypatch):
    """The records give bytes while every source they name is unchanged and
    null as soon as one changes (the counters then describe another kernel)."""
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    step = json.loads((root / "profiles" / "traffic_layer_step.txt").read_text())
    score = json.loads((root / "profiles" / "traffic_score_kernel.txt").read_text())
    # records written for the copied sources (the committed ones) give their bytes
    import hashlib
    h = hashlib.sha256()
    for name in sorted(step["sources"]):
        h.update((root / "long_context_decoding_b200" / "csrc" / name).read_bytes())
    if h.hexdigest() == step["sources_sha256"]:
        assert bench.step_dram_traffic()["bytes_per_layer_step"] == step["dram_bytes_per_layer_step"]
    src = root / "long_context_decoding_b200" / "csrc" / "score.cu"
    if hashlib.sha256(src.read_bytes()).hexdigest() == score["score_kernel"]["source_sha256"]:
        assert bench.score_traffic()[0] == score["score_kernel"]["dram_bytes_per_launch"]
    # any change to a named source voids both
    src.write_bytes(src.read_bytes() + b"\n// changed\n")
    assert bench.step_dram_traffic() is None
    assert bench.score_traffic() == (None, None)


def test_traffic_records_rehashed_after_a_change(tmp_path, monkeypatch):
    """A record whose hashes are recomputed over the current sources reads back."""
    import hashlib
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    p = root / "profiles" / "traffic_layer_step.txt"
    rec = json.loads(p.read_text())
    h = hashlib.sha256()
    for name in sorted(rec["sources"]):
        h.update((root / "long_context_decoding_b200" / "csrc" / name).read_bytes())
    rec["sources_sha256"] = h.hexdigest()
    rec["dram_bytes_per_layer_step"] = 123.0
    p.write_text(json.dumps(rec))
    assert bench.step_dram_traffic()["bytes_per_layer_step"] == 123.0


def test_planted_recall():
    sel = np.array([[[1, 5, 9, 0], [2, 4, 0, 0]]])
    nsel = np.array([[3, 2]])
    planted = np.array([[[5, 9], [4, 7]]])
    r = bench.planted_recall(sel, nsel, planted)
    assert r["per_unit"] == [1.0, 0.5] and r["mean"] == 0.75 and r["min"] == 0.5
    # entries past n_sel do not count
    r = bench.planted_recall(sel, np.array([[1, 2]]), planted)
    assert r["per_unit"][0] == 0.0
