"""Pins of the oracle's chunk-aware masks and compact key index (CPU only)."""

import json
import os

import numpy as np
import pytest

from oracle import chunks, mask, scalar

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _random_starts(rng, n):
    kind = rng.integers(3)
    if kind == 0:
        P = int(rng.integers(1, 9))
        return chunks.uniform_starts(n, P, 0), P
    if kind == 1:
        P = int(rng.integers(2, 9))
        return chunks.uniform_starts(n, P, int(rng.integers(0, P))), P
    return chunks.varlen_starts(rng.integers(1, 12, size=n + 1).tolist(), n), None


@pytest.mark.parametrize("seed", range(4))
def test_dense_mask_matches_scalar_definition(seed):
    rng = np.random.default_rng(seed)
    for _ in range(10):
        n = int(rng.integers(1, 24))
        starts, _ = _random_starts(rng, n)
        L = int(rng.integers(0, n + 2))
        for mode in mask.MODES:
            M = mask.dense_mask(n, starts, L, mode)
            S = np.array([[scalar.in_mask(i, j, set(starts.tolist()), n, L, mode) for j in range(n)] for i in range(n)])
            assert np.array_equal(M, S)


def test_compact_index_expands_to_the_dense_mask():
    """300 random cases: uniform, cyclic, variable chunks; L from 0 to beyond n; both masks."""
    rng = np.random.default_rng(123)
    for _ in range(300):
        n = int(rng.integers(1, 70))
        starts, _ = _random_starts(rng, n)
        L = int(rng.integers(0, n + 3))
        mode = mask.MODES[int(rng.integers(2))]
        ls, nbb, bpos = mask.compact_index(n, starts, L, mode)
        assert np.array_equal(mask.expand_compact(n, ls, nbb, bpos), mask.dense_mask(n, starts, L, mode))
        assert np.all(np.diff(ls) >= 0) and np.all(np.diff(nbb) >= 0)
        assert np.all(ls <= np.arange(n) + 1)


@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("L", [0, 1, 3, 4, 5, 11])
def test_key_count_closed_forms(P, L):
    """Uniform chunks, offset 0:
    M_train: |S(i)| = floor(i/P) + (i mod P) + 1  when L <= (i mod P) + 1;
    M_test : |S(i)| = max(0, floor((i-L+1)/P)) + min(L, i+1),
             except L = 0 at i = n-1 with n mod P != 0, where the cut last chunk adds one.
    """
    for n in (1, 7, 33, 64, 100):
        starts = chunks.uniform_starts(n, P, 0)
        ct = mask.key_counts(n, starts, L, "train")
        cs = mask.key_counts(n, starts, L, "test")
        for i in range(n):
            if L <= (i % P) + 1:
                assert ct[i] == i // P + (i % P) + 1
            expect = max(0, (i - L + 1) // P) + min(L, i + 1)
            if L == 0 and i == n - 1 and n % P != 0:
                expect += 1
            assert cs[i] == expect, (n, i)


def test_page_worked_count_n1024_P4_L32():
    g = json.load(open(os.path.join(GOLDEN, "page_kv_count.json")))
    n, P, L = g["n"], g["P"], g["L"]
    starts = chunks.uniform_starts(n, P, 0)
    counts = mask.key_counts(n, starts, L, g["mode"])
    assert n // P + L == g["page_value_roughly"]
    assert counts[-1] == g["exact_last_query_keys"]
    assert counts[-1] == n // P + L - L // P
    assert counts.max() <= g["page_value_roughly"]


def test_page_compression_P8_L64():
    g = json.load(open(os.path.join(GOLDEN, "page_compression.json")))
    n, P, L = g["n_check"], g["P"], g["L"]
    starts = chunks.uniform_starts(n, P, 0)
    row = mask.mask_row(n - 1, n, starts, L, "test")
    assert row.sum() == g["entries_at_n_check"]
    assert abs(n / row.sum() - g["compression_roughly"]) < 0.5


def test_special_cases_reduce_to_causal():
    for n in (5, 17, 40):
        causal = np.tril(np.ones((n, n), dtype=bool))
        # P = 1: every token is a completed chunk
        for mode in mask.MODES:
            assert np.array_equal(mask.dense_mask(n, chunks.uniform_starts(n, 1), 0, mode), causal)
        # L >= n: the window already covers every earlier token
        for P in (2, 4, 8):
            for mode in mask.MODES:
                assert np.array_equal(mask.dense_mask(n, chunks.uniform_starts(n, P, 1), n, mode), causal)
        # one chunk covering the sequence with M_train: causal
        assert np.array_equal(mask.dense_mask(n, np.array([0]), 0, "train"), causal)


def test_test_mask_within_train_mask_and_equal_for_wide_window():
    rng = np.random.default_rng(9)
    for _ in range(50):
        n = int(rng.integers(2, 60))
        starts = chunks.varlen_starts(rng.integers(1, 9, size=n).tolist(), n)
        L = int(rng.integers(0, 10))
        Mtr = mask.dense_mask(n, starts, L, "train")
        Mte = mask.dense_mask(n, starts, L, "test")
        assert not np.any(Mte & ~Mtr)
        maxlen = int(np.max(np.diff(np.append(starts, n))))
        assert np.array_equal(mask.dense_mask(n, starts, maxlen, "test"), mask.dense_mask(n, starts, maxlen, "train"))


def test_test_mask_is_causal_in_the_chunk_sense():
    """No query reads the end state of its own unfinished chunk unless it is in the window."""
    n, P, L = 64, 8, 3
    starts = chunks.uniform_starts(n, P, 0)
    M = mask.dense_mask(n, starts, L, "test")
    end = chunks.chunk_end_of(starts, n)
    for i in range(n):
        assert not np.any(M[i, i + 1:])
        if end[i] != i:
            assert not M[i, end[i]]


def test_mask_row_matches_dense():
    rng = np.random.default_rng(4)
    n = 57
    starts = chunks.varlen_starts(rng.integers(2, 9, size=n).tolist(), n)
    for mode in mask.MODES:
        M = mask.dense_mask(n, starts, 5, mode)
        for i in range(n):
            assert np.array_equal(mask.mask_row(i, n, starts, 5, mode), M[i])
