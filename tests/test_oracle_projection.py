"""Pins of the oracle's projections (CPU only)."""

import numpy as np
import pytest

from oracle import projection, scalar


def test_project_equals_scalar_loop():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 7))
    W = rng.standard_normal((3, 7))
    np.testing.assert_allclose(projection.project(x, W), np.array(scalar.project(x.tolist(), W.tolist())),
                               rtol=1e-13, atol=1e-13)


def test_project_identity_and_orientation():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 6))
    np.testing.assert_array_equal(projection.project(x, np.eye(6)), x)
    # W is (output features, input features): a 2 x 6 selector picks input columns 1 and 4
    sel = np.zeros((2, 6))
    sel[0, 1] = sel[1, 4] = 1
    np.testing.assert_array_equal(projection.project(x, sel), x[:, [1, 4]])


def test_stacked_weights_split_into_the_separate_projections():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 16))
    Ws = [rng.standard_normal((w, 16)) for w in (16, 16, 8, 8)]
    parts = projection.split(projection.project(x, np.concatenate(Ws)), [16, 16, 8, 8])
    for p, W in zip(parts, Ws):
        np.testing.assert_allclose(p, x @ W.T, rtol=1e-13, atol=1e-13)
    with pytest.raises(ValueError):
        projection.split(projection.project(x, Ws[0]), [8])
