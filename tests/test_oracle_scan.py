"""Pins of the oracle's selective scan (CPU only).

Each test checks the oracle against something other than itself: the literal
scalar loop, closed forms, the chunk-independence the pages state, and a
library routine (numpy convolution, torch softplus).
"""

import numpy as np
import pytest
import torch

from oracle import chunks, scalar, ssm



def _rand_case(rng, T, D, N):
    u = rng.standard_normal((T, D))
    dt = rng.standard_normal((T, D)) - 2.0
    bias = rng.uniform(-3, 0, D)
    A = -np.exp(rng.uniform(0, np.log(16), (D, N)))
    Bm = rng.standard_normal((T, N))
    Cm = rng.standard_normal((T, N))
    return u, dt, bias, A, Bm, Cm


@pytest.mark.parametrize("seed", range(6))
def test_scan_matches_scalar_loop(seed):
    rng = np.random.default_rng(seed)
    T, D, N = 13, 3, 4
    u, dt, bias, A, Bm, Cm = _rand_case(rng, T, D, N)
    starts = sorted({0} | set(rng.choice(np.arange(1, T), size=3, replace=False).tolist()))
    is_start = chunks.is_start_mask(starts, T)
    y, _ = ssm.selective_scan(u, dt, bias, A, Bm, Cm, is_start)
    ys = scalar.scan(u.tolist(), dt.tolist(), bias.tolist(), A.tolist(), Bm.tolist(), Cm.tolist(), set(starts))
    np.testing.assert_allclose(y, np.array(ys), rtol=1e-12, atol=1e-13)


def test_softplus_matches_library():
    z = np.linspace(-30, 40, 1001)
    ref = torch.nn.functional.softplus(torch.tensor(z, dtype=torch.float64), beta=1.0, threshold=20.0).numpy()
    np.testing.assert_allclose(ssm.softplus(z), ref, rtol=1e-14, atol=1e-300)
    assert abs(ssm.softplus(0.0) - np.log(2.0)) < 1e-15


def test_chunk_size_one_is_a_per_token_map_independent_of_A():
    """P = 1: every token restarts the state, so y = delta * u * (B . C), whatever A is."""
    rng = np.random.default_rng(1)
    T, D, N = 40, 5, 16
    u, dt, bias, A, Bm, Cm = _rand_case(rng, T, D, N)
    is_start = np.ones(T, dtype=bool)
    y, _ = ssm.selective_scan(u, dt, bias, A, Bm, Cm, is_start)
    delta = ssm.softplus(dt + bias)
    closed = delta * u * (Bm * Cm).sum(axis=1)[:, None]
    np.testing.assert_allclose(y, closed, rtol=1e-12, atol=1e-14)
    y2, _ = ssm.selective_scan(u, dt, bias, A * 3.7, Bm, Cm, is_start)
    assert np.array_equal(y, y2)


def test_single_chunk_geometric_convolution():
    """One chunk, constant delta/B/C, scalar A: y_t = C B delta sum_{s<=t} exp(A delta (t-s)) u_s."""
    rng = np.random.default_rng(2)
    T, D, N = 64, 3, 1
    u = rng.standard_normal((T, D))
    z = np.array([-2.0, -1.0, 0.5])
    dt = np.tile(z, (T, 1))
    bias = np.zeros(D)
    A = np.array([[-0.7], [-3.0], [-0.1]])
    Bm = np.full((T, N), 1.3)
    Cm = np.full((T, N), -0.4)
    is_start = np.zeros(T, dtype=bool)
    is_start[0] = True
    y, _ = ssm.selective_scan(u, dt, bias, A, Bm, Cm, is_start)
    delta = ssm.softplus(z)
    for d in range(D):
        kern = np.exp(A[d, 0] * delta[d] * np.arange(T))
        conv = np.convolve(u[:, d], kern)[:T]
        np.testing.assert_allclose(y[:, d], -0.4 * 1.3 * delta[d] * conv, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("seed", range(4))
def test_locality_changes_stay_inside_the_chunk(seed):
    """Perturbing token j moves the output only at positions [j, end(j)] (chunks are independent)."""
    rng = np.random.default_rng(10 + seed)
    T, D, N = 37, 4, 8
    u, dt, bias, A, Bm, Cm = _rand_case(rng, T, D, N)
    starts = chunks.varlen_starts(rng.integers(2, 9, size=40).tolist(), T)
    is_start = chunks.is_start_mask(starts, T)
    end = chunks.chunk_end_of(starts, T)
    y, _ = ssm.selective_scan(u, dt, bias, A, Bm, Cm, is_start)
    for j in rng.choice(T, size=6, replace=False):
        for which in ("u", "dt", "B"):
            u2, dt2, B2 = u.copy(), dt.copy(), Bm.copy()
            {"u": u2, "dt": dt2, "B": B2}[which][j] += 0.5
            y2, _ = ssm.selective_scan(u2, dt2, bias, A, B2, Cm, is_start)
            changed = np.any(np.abs(y2 - y) > 0, axis=1)
            outside = np.ones(T, dtype=bool)
            outside[j: end[j] + 1] = False
            assert not changed[outside].any(), (which, j)
            assert changed[j]


def test_whole_sequence_equals_chunks_scanned_separately():
    rng = np.random.default_rng(5)
    T, D, N = 50, 3, 5
    u, dt, bias, A, Bm, Cm = _rand_case(rng, T, D, N)
    starts = chunks.uniform_starts(T, 8, offset=3)
    assert list(starts[:3]) == [0, 3, 11]
    y, _ = ssm.selective_scan(u, dt, bias, A, Bm, Cm, chunks.is_start_mask(starts, T))
    bounds = list(starts) + [T]
    for a, b in zip(bounds[:-1], bounds[1:]):
        yc, _ = ssm.selective_scan(u[a:b], dt[a:b], bias, A, Bm[a:b], Cm[a:b], np.eye(1, b - a, 0, dtype=bool)[0])
        np.testing.assert_allclose(y[a:b], yc, rtol=0, atol=0)


def test_planted_missing_reset_is_caught():
    """A scan that forgets the chunk reset fails the locality pin (mistake planted in a copy of the oracle)."""
    rng = np.random.default_rng(7)
    T, D, N = 24, 2, 4
    u, dt, bias, A, Bm, Cm = _rand_case(rng, T, D, N)
    starts = chunks.uniform_starts(T, 4)
    no_reset = np.zeros(T, dtype=bool)
    no_reset[0] = True
    y, _ = ssm.selective_scan(u, dt, bias, A, Bm, Cm, no_reset)
    u2 = u.copy()
    u2[1] += 1.0
    y2, _ = ssm.selective_scan(u2, dt, bias, A, Bm, Cm, no_reset)
    end = chunks.chunk_end_of(starts, T)
    assert np.any(np.abs(y2 - y)[end[1] + 1:] > 0)


def test_uniform_and_varlen_starts():
    assert chunks.uniform_starts(10, 4, 0).tolist() == [0, 4, 8]
    assert chunks.uniform_starts(10, 4, 3).tolist() == [0, 3, 7]
    assert chunks.uniform_starts(10, 4, 7).tolist() == [0, 3, 7]
    assert chunks.varlen_starts([3, 5, 9], 10).tolist() == [0, 3, 8]
    assert chunks.boundary_positions([0, 3, 8], 10).tolist() == [2, 7, 9]
    assert chunks.chunk_end_of([0, 3, 8], 10).tolist() == [2, 2, 2, 7, 7, 7, 7, 7, 9, 9]


def test_two_token_chunk_closed_form_separates_B_from_C():
    """Chunk [t0, t1]: y_1 = sum_n C1_n (exp(delta_1 A_n) delta_0 u_0 B0_n + delta_1 u_1 B1_n).

    This pins which projection feeds the state (B) and which reads it (C), and
    that the decay of step t uses that step's own delta.
    """
    rng = np.random.default_rng(11)
    D, N = 3, 6
    u, dt, bias, A, Bm, Cm = _rand_case(rng, 2, D, N)
    is_start = np.array([True, False])
    y, h = ssm.selective_scan(u, dt, bias, A, Bm, Cm, is_start)
    d0 = ssm.softplus(dt[0] + bias)
    d1 = ssm.softplus(dt[1] + bias)
    h1 = np.exp(d1[:, None] * A) * (d0 * u[0])[:, None] * Bm[0][None, :] + (d1 * u[1])[:, None] * Bm[1][None, :]
    np.testing.assert_allclose(h, h1, rtol=1e-13)
    np.testing.assert_allclose(y[1], h1 @ Cm[1], rtol=1e-13)
    np.testing.assert_allclose(y[0], (d0 * u[0])[:, None] * Bm[0][None, :] @ Cm[0], rtol=1e-13)
    ysw, _ = ssm.selective_scan(u, dt, bias, A, Cm, Bm, is_start)
    assert not np.allclose(ysw[1], y[1])
