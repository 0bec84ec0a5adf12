"""Chunk-aware attention masks (oracle; test infrastructure only).

Sources
-------
* pith.science review, "What carries the argument": M_train (Eq. 5) lets a query
  attend to the last token of each completed chunk and to the tokens of its own
  partial chunk; M_test (Eq. 7) restricts inference attention to chunk
  boundaries; a sliding window of L leading tokens kept uncompressed (Eq. 8) is
  combined with the boundary states.
* pith.science review, "Core claim": a causal mask restricts attention to the
  final state of completed chunks plus the current partial chunk.
* pith.science review, Referee Report, major comment on Eq. (7): as printed, the
  test mask would admit the current chunk's final state; the causal reading
  is that only completed chunks count, the current chunk being reached through
  the leading tokens.
* rohan-paul.com summary, "Solution in this Paper": leading tokens keep recent
  context.

Readings
--------
* Leading tokens are the L most recent positions including the query itself,
  the window (i - L, i]; L = 0 is allowed.
* A position that qualifies twice (a boundary inside the window or the
  current chunk) is one key.
* M_train[i, j] = j <= i and (j == end(j) or chunk(j) == chunk(i) or i - j < L)
  M_test [i, j] = j <= i and (j == end(j) or i - j < L)
  where end(j) is the last position of j's chunk (the last chunk ends at n-1).
"""

import numpy as np

from . import chunks as _ch

MODES = ("train", "test")


def dense_mask(n, starts, L, mode):
    """[n, n] boolean mask written straight from the definition above."""
    if mode not in MODES:
        raise ValueError(mode)
    c = _ch.chunk_of(starts, n)
    end = _ch.chunk_end_of(starts, n)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    causal = j <= i
    boundary = (j == end[None, :])
    window = (i - j) < L
    if mode == "train":
        return causal & (boundary | (c[None, :] == c[:, None]) | window)
    return causal & (boundary | window)


def mask_row(i, n, starts, L, mode):
    """Row i of dense_mask, built the same way but for one query (for large n)."""
    c = _ch.chunk_of(starts, n)
    end = _ch.chunk_end_of(starts, n)
    j = np.arange(n)
    causal = j <= i
    boundary = j == end
    window = (i - j) < L
    if mode == "train":
        return causal & (boundary | (c == c[i]) | window)
    return causal & (boundary | window)


def compact_index(n, starts, L, mode):
    """Canonical compact form of the same key sets, one sequence.

    S(i) = {bpos[k] : k < nbb(i)}  united with  [ls(i), i], where
      ls(i) = max(0, min(start(i), i - L + 1))   under M_train,
      ls(i) = max(0, i - L + 1)                  under M_test,
      bpos  = the chunk-end positions in increasing order,
      nbb(i)= the number of bpos strictly below ls(i).
    Every position in [ls(i), i] is in the mask (own chunk or window), and below
    ls(i) only completed-chunk ends qualify, so this is the same set; the tests
    expand it and compare with ``dense_mask`` element by element.
    Returns (ls [n], nbb [n], bpos [n_chunks]) as int64.
    """
    i = np.arange(n)
    if mode == "train":
        start = _ch.chunk_start_of(starts, n)
        ls = np.maximum(0, np.minimum(start, i - L + 1))
    elif mode == "test":
        ls = np.maximum(0, i - L + 1)
    else:
        raise ValueError(mode)
    bpos = _ch.boundary_positions(starts, n)
    nbb = np.searchsorted(bpos, ls, side="left")
    return ls.astype(np.int64), nbb.astype(np.int64), bpos.astype(np.int64)


def expand_compact(n, ls, nbb, bpos):
    """Dense [n, n] mask from a compact index (used to compare encodings)."""
    m = np.zeros((n, n), dtype=bool)
    for i in range(n):
        m[i, bpos[: nbb[i]]] = True
        if ls[i] <= i:
            m[i, ls[i]: i + 1] = True
    return m


def key_counts(n, starts, L, mode):
    """|S(i)| for every query, from the dense definition."""
    return dense_mask(n, starts, L, mode).sum(axis=1)
