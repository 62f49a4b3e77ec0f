"""The benchmark's tile accounting for window heads, on the host: the
separable per-axis count of visited tiles equals the oracle's count of
non-empty tiles (boundary + full) built from the token x token mask."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from gen import config  # noqa: E402
from oracle import bsa_oracle as O  # noqa: E402


@pytest.mark.parametrize("over", [{}, {"prefix": (70,), "T": 8, "H": 8, "W": 12, "T_valid": 8,
                                       "H_valid": 8, "W_valid": 12}])
def test_window_tile_count_matches_oracle_classes(over):
    cfg = config("tiny", **over)
    geo = O.Geometry(cfg)
    perm = O.fixed_perm(geo)
    wins = [(0, -1, -1), (1, -1, -1), (-1, 2, 2), (2, 0, 5), (-1, -1, -1), (4, 3, -1)]
    for w in wins:
        classes = O.tile_classes(geo, perm, w)
        want = cfg["B"] * int((classes > 0).sum())
        assert bench.window_tiles(cfg, [w]) == want, w


def test_window_patterns_cycle_over_heads():
    cfg = config("720p")
    wins = bench.window_heads(cfg, "mixed")
    assert len(wins) == 24 and wins[0] == (1, -1, -1) and wins[1] == (-1, 2, 2)
    assert bench.window_tiles(cfg, wins) < bench.dense_tiles(cfg)
