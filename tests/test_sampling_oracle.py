"""Pins of the oracle's seeded row choice (oracle/sampling.py), on the CPU.

SplitMix64 is checked against outputs published with the generator's reference
implementation; Floyd's algorithm against what it must give whatever the
generator: distinct rows in range, every K-subset equally likely, and the
closed cases K = N and K = 1.
"""
import itertools
from collections import Counter

import numpy as np
import pytest

from oracle import sampling


def test_splitmix64_published_outputs():
    # started at state 0: the first four outputs of the reference generator
    assert [sampling.splitmix64(0, i) for i in range(4)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]
    # started at state 1234567 (the reference implementation's test seed)
    assert [sampling.splitmix64(1234567, i) for i in range(3)] == [
        6457827717110365317, 3203168211198807973, 9817491932198370423]


@pytest.mark.parametrize("N,K", [(10, 3), (1000, 1000), (5, 1), (10_000_000, 4096)])
def test_rows_distinct_and_in_range(N, K):
    rows = sampling.floyd_rows(N, K, 7)
    assert len(rows) == K and len(set(rows)) == K
    assert all(0 <= r < N for r in rows)


def test_k_equals_n_takes_every_row_and_k1_is_uniform():
    assert sorted(sampling.floyd_rows(50, 50, 3)) == list(range(50))
    counts = Counter(sampling.floyd_rows(6, 1, s)[0] for s in range(6000))
    assert set(counts) == set(range(6))
    chi2 = sum((c - 1000) ** 2 / 1000 for c in counts.values())
    assert chi2 < 20.5  # 5 degrees of freedom, p < 0.001


def test_every_subset_equally_likely():
    """N = 6, K = 3: 20 subsets over 20,000 seeds; chi-square with 19 degrees of
    freedom below its 0.999 quantile (43.8)."""
    counts = Counter(frozenset(sampling.floyd_rows(6, 3, s)) for s in range(20_000))
    subsets = {frozenset(c) for c in itertools.combinations(range(6), 3)}
    assert set(counts) == subsets
    chi2 = sum((counts[s] - 1000) ** 2 / 1000 for s in subsets)
    assert chi2 < 43.8


def test_rejection_keeps_small_ranges_uniform():
    st = sampling._Stream(11)
    draws = np.array([st.below(3) for _ in range(30_000)])
    freq = np.bincount(draws, minlength=3) / len(draws)
    assert np.all(np.abs(freq - 1 / 3) < 0.01)


def test_planted_mistakes_are_caught(monkeypatch):
    """A wrong multiplier, a missing rejection step, or taking t instead of j on a
    repeat each break one of the pins above."""
    good = sampling.splitmix64
    monkeypatch.setattr(sampling, "GAMMA", sampling.GAMMA ^ 2)
    assert sampling.splitmix64(0, 0) != 0xE220A8397B1DCDAF
    monkeypatch.setattr(sampling, "GAMMA", 0x9E3779B97F4A7C15)
    assert good(0, 0) == 0xE220A8397B1DCDAF

    def floyd_repeat_t(N, K, seed):
        st = sampling._Stream(seed)
        taken, rows = set(), []
        for j in range(N - K, N):
            t = st.below(j + 1)
            taken.add(t)
            rows.append(t)
        return rows

    assert any(len(set(floyd_repeat_t(6, 3, s))) < 3 for s in range(200))
