"""Selective state-space scan that replaces W_K and W_V (oracle; test infrastructure only).

Sources
-------
* rohan-paul.com summary, "Solution in this Paper": SSM blocks replace the key
  and value projection matrices and compress several tokens into one state.
* pith.science review, "Core claim": K^(p) = SSM_K(X^(p)), V^(p) = SSM_V(X^(p))
  for each chunk p; two separate SSMs.
* pith.science review, "Assumptions & free parameters": the SSM is a selective
  state-space model (Mamba, Section 3.2, Eq. 3).
* pith.science review, "What carries the argument": one state per chunk of P
  tokens, i.e. the recurrence restarts at every chunk start.

Readings taken where the pages are silent (Eq. 3 itself is not reproduced)
--------------------------------------------------------------------------
* Mamba's selective SSM with a diagonal A (D x N, A < 0): for token t and
  channel d,  delta = softplus(dt[t, d] + dt_bias[d]);
  h[d, :] <- exp(delta * A[d, :]) * h[d, :] + delta * u[t, d] * B[t, :];
  y[t, d] = sum_n C[t, n] * h[d, n].  Zero-order hold for A, Euler step for B.
  No skip term D, no convolution and no gate inside the block.  The SSM input
  u is the layer input x (width d_model = H * head_dim).
* B and C are per token and shared by all channels; each SSM has its own
  dt, dt_bias, A, B, C.
* h = 0 at every chunk start (taken before the update of that token).
* softplus(z) = z for z > 20, else log1p(exp(z)).
"""

import numpy as np


def softplus(z):
    z = np.asarray(z, dtype=np.float64)
    return np.where(z > 20.0, z, np.log1p(np.exp(np.minimum(z, 20.0))))


def selective_scan(u, dt, dt_bias, A, Bm, Cm, is_start, h0=None):
    """Naive per-token recurrence over a flattened token axis.

    u, dt   : [T, D]  layer input and pre-softplus step
    dt_bias : [D]
    A       : [D, N]  (negative)
    Bm, Cm  : [T, N]
    is_start: [T] bool, True where a chunk begins (sequence starts included)
    h0      : optional [D, N] state before token 0 (used only if token 0 is not a start)

    Returns (y [T, D], h_last [D, N]) in float64.
    """
    u = np.asarray(u, dtype=np.float64)
    dt = np.asarray(dt, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    Cm = np.asarray(Cm, dtype=np.float64)
    b = np.asarray(dt_bias, dtype=np.float64)
    T, D = u.shape
    N = A.shape[1]
    h = np.zeros((D, N)) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.zeros((T, D))
    for t in range(T):
        delta = softplus(dt[t] + b)                      # [D]
        if is_start[t]:
            h = np.zeros((D, N))
        h = np.exp(delta[:, None] * A) * h + (delta * u[t])[:, None] * Bm[t][None, :]
        y[t] = h @ Cm[t]
    return y, h


def kv_ssm(x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, is_start):
    """Both SSMs over the same input x: returns (K, V) as [T, D] float64."""
    K, _ = selective_scan(x, dt_k, bias_k, A_k, B_k, C_k, is_start)
    V, _ = selective_scan(x, dt_v, bias_v, A_v, B_v, C_v, is_start)
    return K, V
