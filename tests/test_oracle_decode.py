"""Pins of the oracle's decode step: decode equals the M_test prefill row by row (CPU only)."""

import numpy as np
import pytest

from oracle import attention, chunks, decode, mask, ssm


def _params(rng, D, N):
    bias = np.stack([rng.uniform(-4, -1, D) for _ in range(2)])
    A = np.stack([-np.exp(rng.uniform(0, np.log(16), (D, N))) for _ in range(2)])
    return bias, A


@pytest.mark.parametrize("P,offset,L", [(4, 0, 3), (4, 1, 1), (3, 2, 5), (8, 0, 9), (3, 1, 15), (4, 2, 20)])
def test_decode_equals_test_mask_prefill(P, offset, L):
    """A prefill of n0 = 11 tokens handed to the cache, then decoding to n = 20, reproduces the M_test
    prefill rows (the last two cases keep a window longer than the prefill)."""
    rng = np.random.default_rng(P * 100 + offset * 10 + L)
    B, H, dh, N = 2, 2, 4, 5
    D = H * dh
    n0, m = 11, 9
    n = n0 + m
    bias, A = _params(rng, D, N)
    x = rng.standard_normal((B, n, D))
    dt = rng.standard_normal((2, B, n, D)) - 1
    Bm = rng.standard_normal((2, B, n, N))
    Cm = rng.standard_normal((2, B, n, N))
    q = rng.standard_normal((B, n, H, dh))
    scale = 1 / np.sqrt(dh)
    starts = chunks.uniform_starts(n, P, offset)
    is_start = chunks.is_start_mask(starts, n)
    M = mask.dense_mask(n, starts, L, "test")
    K = np.zeros((B, n, D))
    V = np.zeros((B, n, D))
    h_last = np.zeros((2, B, D, N))
    O_pre = np.zeros((B, n, H, dh))
    for b in range(B):
        for s, out in ((0, K), (1, V)):
            y, _ = ssm.selective_scan(x[b], dt[s, b], bias[s], A[s], Bm[s, b], Cm[s, b], is_start)
            out[b] = y
            _, h = ssm.selective_scan(x[b, :n0], dt[s, b, :n0], bias[s], A[s], Bm[s, b, :n0], Cm[s, b, :n0],
                                      is_start[:n0])
            h_last[s, b] = h
        O_pre[b], _ = attention.masked_attention(q[b], K[b].reshape(n, H, dh), V[b].reshape(n, H, dh), M, scale)
    cache = decode.cache_from_prefill(K.reshape(B, n, H, dh)[:, :n0], V.reshape(B, n, H, dh)[:, :n0],
                                      h_last, n0, P, offset, L, H, dh, N)
    for t in range(n0, n):
        o = cache.step(q[:, t], x[:, t], dt[:, :, t], bias, A, Bm[:, :, t], Cm[:, :, t], scale)
        np.testing.assert_allclose(o, O_pre[:, t], rtol=1e-10, atol=1e-12)
        assert cache.n_keys(0, t) == M[t].sum()


def test_chunk_start_end_rule():
    P, o = 4, 3
    starts = chunks.uniform_starts(40, P, o).tolist()
    assert [t for t in range(40) if decode.is_chunk_start(t, P, o)] == starts
    ends = chunks.boundary_positions(starts, 40).tolist()[:-1]
    assert [t for t in range(39) if decode.is_chunk_end(t, P, o)] == ends


def test_decode_key_count_closed_form():
    """With offset 0 the query at position t reads floor((t-L+1)/P) boundaries plus L window tokens."""
    c = decode.DecodeCache(1, 1, 1, 1, 8, 0, 64)
    t = 16384
    c.bpos[0] = [p for p in range(t) if decode.is_chunk_end(p, 8, 0)]
    assert c.n_keys(0, t) == (t - 64 + 1) // 8 + 64 == 2104


def test_decode_rejects_empty_window():
    with pytest.raises(ValueError):
        decode.DecodeCache(1, 1, 1, 1, 4, 0, 0)
