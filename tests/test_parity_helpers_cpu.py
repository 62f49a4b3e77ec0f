"""The near-tie acceptance rule of the parity tests, on the host: which
top-k lists count as correct for a row of fp32 block scores."""
import itertools

import numpy as np

from oracle import bsa_oracle as O
from parity_helpers import TIE_REL, topk_alternatives


def test_no_near_tie_gives_the_oracle_list():
    rng = np.random.default_rng(0)
    for _ in range(50):
        s = rng.normal(size=40).astype(np.float32)
        for k in (1, 5, 39, 40):
            assert topk_alternatives(s, k) == [O.topk_row(s, k)]


def test_exact_tie_at_the_boundary_admits_both():
    s = np.array([5.0, 3.0, 2.0, 3.0, 1.0], dtype=np.float32)
    alts = topk_alternatives(s, 2)
    assert alts == [[0, 1], [0, 3]]
    assert O.topk_row(s, 2) in alts


def test_every_k_subset_by_enumeration():
    """A k-subset is accepted exactly when it keeps every block clearly above
    the k-th score and drops every block clearly below it."""
    rng = np.random.default_rng(1)
    for _ in range(40):
        n = int(rng.integers(4, 10))
        # clustered values so that near ties are common
        s = (rng.integers(0, 4, size=n) + rng.normal(scale=1e-6, size=n)).astype(np.float32)
        k = int(rng.integers(1, n + 1))
        kth = np.sort(s.astype(np.float64))[::-1][k - 1]
        band = TIE_REL * np.abs(s).max()
        want = []
        for sub in itertools.combinations(range(n), k):
            inside = np.zeros(n, dtype=bool)
            inside[list(sub)] = True
            if np.all(inside[s > kth + band]) and not np.any(inside[s < kth - band]):
                want.append(list(sub))
        assert sorted(topk_alternatives(s, k)) == sorted(want)
