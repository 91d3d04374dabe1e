"""The byte model and the cost-model fits of the sweep (host logic)."""
import math

import pytest

from long_context_decoding_b200 import cost


def test_unit_bytes_by_hand():
    # L = 1000, prefix 20, window 50: candidates hold tokens [20, 950): pages 1..59
    u = cost.unit_bytes(1000, 128, 20, 50, 160)
    assert u.candidates == 59 and u.k_pages == 10
    assert u.attended == 20 + 50 + 160
    assert u.meta == 59 * 4 * 128 and u.kv == 230 * 4 * 128
    # every candidate kept: no metadata is read, every token attended
    u = cost.unit_bytes(1000, 128, 20, 50, 16 * 59)
    assert u.meta == 0 and u.attended == 1000
    # prefix and window cover the sequence: no candidates
    u = cost.unit_bytes(60, 128, 20, 50, 160)
    assert u.candidates == 0 and u.attended == 60 and u.meta == 0


def test_path_of():
    assert cost.path_of(65536, 128, 1024, 0) == "prefix_window"
    assert cost.path_of(65536, 128, 1024, 4096) == "one_call"
    assert cost.path_of(4096, 128, 1024, 4096) == "dense"       # 256 pages >= 184 candidates
    assert cost.path_of(4096, 128, 1024, None) == "dense"
    assert cost.path_of(100, 128, 1024, 160) == "prefix_window"  # nothing to select


def test_fit_per_path_recovers_the_model():
    bw = 6.5e12
    t0 = {"prefix_window": 17e-6, "one_call": 23e-6, "dense": 16e-6}
    pts = []
    for path, xs in (("prefix_window", (9e6, 9.5e6, 10e6)),
                     ("one_call", (2e7, 8e7, 1.5e8)), ("dense", (1e8, 5e8, 2e9))):
        for x in xs:
            pts.append({"path": path, "sparse_bytes": x, "sparse_us": 1e6 * (t0[path] + x / bw)})
    f = cost.fit_per_path(pts)
    assert math.isclose(f["bw_gbs"], bw / 1e9, rel_tol=1e-9)
    for k, v in t0.items():
        assert math.isclose(f["t0_us"][k], 1e6 * v, rel_tol=1e-9)
    assert f["max_rel_err"] < 1e-9
