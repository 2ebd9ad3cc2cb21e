"""The bench's accounting of one Newton call (host logic, no GPU): how many
launches of work it makes (the guess launch with up to three fused sweeps,
one launch per further sweep, the iterations launched one by one, and in
tolerance mode the device loop over the rest of the cap as one launch), which
iterations have launches of their own (the ones its per-launch roofline
averages), the algorithmic bytes of a solve, and the stored DRAM-traffic
figures, which are reported only for the kernel sources they were taken on.
"""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from nonlinear_rnn_pararnn_b200 import _lib  # noqa: E402


def test_device_loop_start_matches_the_library_default():
    assert bench.LOOP_FROM == _lib.SLSTM_DEFAULT_LOOP_FROM


def test_guess_and_newton_launch_counts():
    assert bench.guess_launches(0) == 1 and bench.guess_launches(3) == 1
    assert bench.guess_launches(4) == 2 and bench.guess_launches(6) == 4
    # tolerance mode: 2 iterations one by one, then one loop launch over the rest of the cap
    assert bench.newton_launches(2, 16, True) == 1 + 2 + 1
    assert bench.newton_launches(5, 16, True) == 3 + 2 + 1
    # a cap that the separate launches already cover: no loop
    assert bench.newton_launches(2, 2, True) == 1 + 2
    assert bench.newton_launches(2, 1, True) == 1 + 1
    # fixed mode: one launch per iteration
    assert bench.newton_launches(2, 4, False) == 1 + 4


def test_separately_timed_iterations():
    assert bench.separate_iterations(2, True) == 2
    assert bench.separate_iterations(1, True) == 1
    assert bench.separate_iterations(5, True) == 2   # iterations 3..5 ran inside the loop
    assert bench.separate_iterations(5, False) == 5


def test_solve_bytes():
    # guess launch 32 B/elem, each further sweep launch 36, each iteration 48
    assert bench.solve_bytes_per_elem(2, 2) == 32 + 2 * 48
    assert bench.solve_bytes_per_elem(2, 5) == 32 + 2 * 36 + 2 * 48
    assert bench.solve_bytes_per_elem(0, 0) == 32


def test_traffic_reported_only_for_its_sources(monkeypatch):
    sha = bench.newton_sources_sha256()
    monkeypatch.setattr(bench, "NEWTON_TRAFFIC", {"sources_sha256": sha, "guess": 30.0, "sweep": None, "iter": 46.0})
    assert bench.newton_iter_traffic_bytes(1000) == 46000.0
    assert bench.newton_traffic_bytes(1000, 2, 2) == (30.0 + 2 * 46.0) * 1000
    assert bench.newton_traffic_bytes(1000, 2, 5) is None   # a separate sweep launch was not captured
    monkeypatch.setattr(bench, "NEWTON_TRAFFIC", {"sources_sha256": "0" * 64, "guess": 30.0, "sweep": None,
                                                  "iter": 46.0})
    assert bench.newton_iter_traffic_bytes(1000) is None
    assert bench.newton_traffic_bytes(1000, 2, 2) is None
