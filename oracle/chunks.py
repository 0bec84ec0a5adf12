"""Chunk boundaries of one sequence (oracle; test infrastructure only).

Sources
-------
* pith.science review of Attamba, "What carries the argument": the KV-SSM reads
  a chunk of P tokens and yields one state per chunk; cyclic chunking shifts the
  chunk offset by the layer index.
* pith.science review, "Assumptions & free parameters": chunk size P in
  {4, 8, 64, 128}; cyclic chunking layer offset = layer index.
* pith.science review, "If this is right": variable-length chunk boundaries are
  given cu_seqlens-style (prefix offsets of chunk starts).

Readings taken where the pages are silent
-----------------------------------------
* The cyclic offset is o = layer_idx mod P and the chunk starts of a sequence of
  length n are {0} united with {o + kP : k >= 0, 0 < o + kP < n}; when o > 0 the
  first chunk [0, o) is short.  The last chunk is cut at n.
* A sequence start is always a chunk start; chunks never cross sequences.
"""

import numpy as np


def uniform_starts(n, P, offset=0):
    """Sequence-relative chunk starts for uniform chunks of size P shifted by ``offset``."""
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    o = offset % P
    starts = {0}
    s = o
    while s < n:
        if s > 0:
            starts.add(s)
        s += P
    return np.array(sorted(starts), dtype=np.int64)


def varlen_starts(lengths, n):
    """Chunk starts from a list of chunk lengths; the running sum is cut at n."""
    starts = []
    pos = 0
    for ln in lengths:
        if pos >= n:
            break
        starts.append(pos)
        pos += int(ln)
    if not starts or starts[0] != 0:
        raise ValueError("a sequence must start a chunk at position 0")
    return np.array(starts, dtype=np.int64)


def chunk_of(starts, n):
    """c[j]: index (within the sequence) of the chunk holding position j."""
    c = np.zeros(n, dtype=np.int64)
    for k, s in enumerate(starts):
        c[s:] = k
    return c


def chunk_start_of(starts, n):
    """start(j): first position of the chunk holding j."""
    return np.asarray(starts)[chunk_of(starts, n)]


def chunk_end_of(starts, n):
    """end(j): last position of the chunk holding j (the last chunk ends at n - 1)."""
    ends = np.append(np.asarray(starts)[1:], n) - 1
    return ends[chunk_of(starts, n)]


def boundary_positions(starts, n):
    """Positions that end a chunk, in increasing order (one per chunk)."""
    return np.append(np.asarray(starts)[1:], n) - 1


def is_start_mask(starts, n):
    m = np.zeros(n, dtype=bool)
    m[np.asarray(starts)] = True
    return m


def flatten_batch(starts_per_seq, n):
    """cu over B sequences of length n laid end to end: chunk starts plus the final B*n."""
    cu = []
    for b, st in enumerate(starts_per_seq):
        cu.extend((b * n + np.asarray(st)).tolist())
    cu.append(len(starts_per_seq) * n)
    return np.array(cu, dtype=np.int64)
