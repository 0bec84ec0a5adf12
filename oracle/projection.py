"""The layer's projections (oracle; test infrastructure only).

Sources
-------
* pith.science review, "Core claim": the SSMs stand in for the key and value
  projections W_K and W_V; the query projection and the output projection stay.
* pith.science review, "Assumptions & free parameters": the SSM is Mamba's
  selective SSM (Eq. 3), whose step Delta and matrices B, C depend on the input,
  i.e. are projections of it.

Reading
-------
* Every projection is a plain linear map without bias, y = x W^T with W stored as
  (output features, input features).  The input projections are stacked along
  their output features into one matrix; column segments of the product are the
  individual outputs (q, dt_K, dt_V, B_K, C_K, B_V, C_V).
"""

import numpy as np


def project(x, W):
    """y = x W^T in float64.  x: [M, K], W: [Nout, K] -> [M, Nout]."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def split(y, widths):
    """Column segments of y, in order, of the given widths (must sum to y's width)."""
    out, c = [], 0
    for w in widths:
        out.append(y[:, c:c + w])
        c += w
    if c != y.shape[1]:
        raise ValueError("segment widths do not cover the output")
    return out
