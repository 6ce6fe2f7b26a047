"""Pins for the oracle's expert -> rank partition (CPU only).

The oracle fills ranks with a loop; these tests check it against what the
TensorRT-LLM PR #13888 pages fix: the base/remainder examples in its commit
messages and review thread (tests/golden/partition_examples.txt), the
closed-form rank lookup its divisible-fast-path commit describes (base and
remainder hoisted, ``expert // base`` when the remainder is zero), and the
structural facts of a ceil/floor contiguous split.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "partition_examples.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            E, R, base, rem = map(int, parts[:4])
            rest = parts[4:]
            rows.append((E, R, base, rem, rest))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: f"E{r[0]}_R{r[1]}")
def test_golden_examples(oracle_mod, row):
    E, R, base, rem, rest = row
    # the printed base/remainder are E // R and E % R
    assert (E // R, E % R) == (base, rem)
    if rest == ["ERROR_EMPTY_RANK"]:
        with pytest.raises(oracle_mod.OracleError) as ei:
            oracle_mod.partition(E, R)
        assert ei.value.code == oracle_mod.EMPTY_RANK
        return
    first = oracle_mod.partition(E, R)
    sizes = np.diff(first)
    if rest == ["-"]:
        expect = [base + 1] * rem + [base] * (R - rem)
    else:
        expect = [int(v) for v in rest]
    assert sizes.tolist() == expect
    assert first[0] == 0 and first[-1] == E


def _rank_closed_form(e, E, R):
    """The rank lookup as the divisible-fast-path commit describes it."""
    base, rem = E // R, E % R
    if rem == 0:
        return e // base
    if e < rem * (base + 1):
        return e // (base + 1)
    return rem + (e - rem * (base + 1)) // base


def test_exhaustive_structure_and_closed_form(oracle_mod):
    for E in range(1, 257):
        for R in range(1, E + 1):
            first = oracle_mod.partition(E, R)
            sizes = np.diff(first)
            assert first[0] == 0 and first[-1] == E
            assert sizes.min() >= 1
            assert sizes.max() - sizes.min() <= 1
            assert np.all(np.diff(sizes) <= 0), "larger ranks come first"
            rank_of = np.repeat(np.arange(R), sizes)
            cf = np.array([_rank_closed_form(e, E, R) for e in range(E)])
            assert np.array_equal(rank_of, cf), (E, R)


def test_sparse_large_range(oracle_mod):
    rng = np.random.default_rng(7)
    for _ in range(300):
        E = int(rng.integers(1, 4097))
        R = int(rng.integers(1, E + 1))
        first = oracle_mod.partition(E, R)
        sizes = np.diff(first)
        assert sizes.sum() == E and sizes.max() - sizes.min() <= 1
        assert int((sizes == sizes.max()).sum()) == (E % R if E % R else R)


@pytest.mark.parametrize("E,R", [(1, 2), (3, 4), (7, 8), (2, 8), (0, 1), (5, 0)])
def test_refusals(oracle_mod, E, R):
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.partition(E, R)
    if E >= 1 and R >= 1:
        assert ei.value.code == oracle_mod.EMPTY_RANK
    else:
        assert ei.value.code == oracle_mod.INVALID_ARG
