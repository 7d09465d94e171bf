"""Pins of the IVF inverted-list oracle (oracle/ivf.py), on the CPU.

The rule ("Flash-GMM" abstract: border vectors filed under several clusters,
read as: always the rank-1 list, the rank-j list when r_j >= tau) is pinned by
things other than the oracle's own formula:

  * a case worked by hand;
  * tau above 1 reduces the index to a plain partition by the rank-1 label,
    checked against per-label np.flatnonzero;
  * tau = 0 files every point under all m of its components, checked against
    Python set membership;
  * invariants on random input: every point exactly once in its rank-1 list,
    lists ascending, the total equal to N plus the kept entries of rank >= 2;
  * the threshold is decided in float32, like the kernel's float tau.

The mutant test at the end plants plausible mistakes in a copy of the oracle
and checks that some pin fails for each.
"""
import inspect
import types

import numpy as np
import pytest

from oracle import ivf
from soft_clustering_em_b200 import synth


def _lists(offsets, ids):
    return [ids[offsets[k]:offsets[k + 1]].tolist() for k in range(len(offsets) - 1)]


def pin_hand_worked(f):
    # K = 3, m = 2, tau = 0.3.  Rank-1 lists: point 0 -> 2, 1 -> 0, 2 -> 1, 3 -> 2.
    # Rank 2: point 0 (0.4 >= 0.3) also joins list 0; point 1 (0.05) does not join 1;
    # point 2 (0.5) joins 2; point 3 (0.3, equal to tau) joins 1.
    idx = np.array([[2, 0], [0, 1], [1, 2], [2, 1]])
    resp = np.array([[0.6, 0.4], [0.9, 0.05], [0.5, 0.5], [0.7, 0.3]], dtype=np.float32)
    offsets, ids = f(idx, resp, 3, 0.3)
    assert offsets.tolist() == [0, 2, 4, 7]
    assert _lists(offsets, ids) == [[0, 1], [2, 3], [0, 2, 3]]


def pin_hard_partition(f):
    idx, resp = synth.topm_inputs(5_000, 37, 3, seed=11)
    offsets, ids = f(idx, resp, 37, 1.5)
    assert offsets[-1] == 5_000
    for k, got in enumerate(_lists(offsets, ids)):
        assert got == np.flatnonzero(idx[:, 0] == k).tolist()


def pin_all_entries(f):
    idx, resp = synth.topm_inputs(400, 9, 4, seed=12)
    offsets, ids = f(idx, resp, 9, 0.0)
    assert offsets[-1] == 400 * 4
    for k, got in enumerate(_lists(offsets, ids)):
        assert got == [n for n in range(400) if k in set(idx[n].tolist())]


def pin_invariants(f):
    N, K, m, tau = 3_001, 64, 3, 0.05
    idx, resp = synth.topm_inputs(N, K, m, seed=13, ties_at=tau)
    offsets, ids = f(idx, resp, K, tau)
    kept = int((resp[:, 1:] >= np.float32(tau)).sum())
    assert offsets[0] == 0 and np.all(np.diff(offsets) >= 0)
    assert offsets[-1] == len(ids) == N + kept
    seen_top = np.zeros(N, dtype=np.int64)
    for k, lst in enumerate(_lists(offsets, ids)):
        assert lst == sorted(set(lst))  # ascending, no point twice
        for n in lst:
            j = int(np.flatnonzero(idx[n] == k)[0])  # the point's rank for this list
            assert j == 0 or resp[n, j] >= np.float32(tau)
            seen_top[n] += j == 0
    assert np.all(seen_top == 1)


def pin_float32_threshold(f):
    r = np.float32(0.1)  # 0.10000000149...
    tau = 0.1000000018  # above r in float64, but float32(tau) == r
    assert np.float64(r) < tau and np.float32(tau) == r
    idx = np.array([[0, 1], [1, 0]])
    resp = np.array([[0.8, r], [0.9, np.nextafter(r, np.float32(0))]], dtype=np.float32)
    offsets, ids = f(idx, resp, 2, tau)
    # point 0: list 0 (rank 1) and list 1 (r == float32(tau)); point 1: list 1 only
    assert _lists(offsets, ids) == [[0], [0, 1]]


PINS = [pin_hand_worked, pin_hard_partition, pin_all_entries, pin_invariants,
        pin_float32_threshold]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_meets_pin(pin):
    pin(ivf.ivf_lists)


MUTANTS = {
    "strict_threshold": ("(resp >= np.float32(tau))", "(resp > np.float32(tau))"),
    "no_rank_one_rule": ("keep = rank_one | (resp", "keep = (resp"),
    "last_rank_forced": ("rank_one[:, 0] = True", "rank_one[:, -1] = True"),
    "points_descending": ("np.lexsort((points, lists))", "np.lexsort((-points, lists))"),
    "offsets_shifted": ("offsets[1:] = np.cumsum", "offsets[:-1] = np.cumsum"),
    "threshold_in_f64": ("(resp >= np.float32(tau))", "(resp >= np.float64(tau))"),
}


def _mutant(name):
    src = inspect.getsource(ivf)
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType("ivf_" + name)
    exec(compile(src.replace(old, new), "ivf_" + name, "exec"), mod.__dict__)
    return mod.ivf_lists


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    f = _mutant(name)
    caught = 0
    for pin in PINS:
        try:
            pin(f)
        except (AssertionError, IndexError, ValueError):
            caught += 1
    assert caught >= 1, f"no pin noticed mutant {name}"


def test_generator_gives_valid_assignments():
    idx, resp = synth.topm_inputs(2_000, 50, 5, seed=3)
    assert idx.dtype == np.int32 and resp.dtype == np.float32
    assert idx.min() >= 0 and idx.max() < 50
    assert all(len(set(r)) == 5 for r in idx.tolist())
    assert np.all(np.diff(resp, axis=1) <= 0) and np.all(resp.sum(1) <= 1 + 1e-6)
