"""Pins of the oracle's masked attention and of the whole layer in its special cases (CPU only)."""

import numpy as np
import pytest
import scipy.special
import torch

from oracle import attention, chunks, mask, scalar, ssm


def _qkv(rng, n, H, dh):
    return (rng.standard_normal((n, H, dh)), rng.standard_normal((n, H, dh)), rng.standard_normal((n, H, dh)))


def test_causal_case_matches_torch_sdpa():
    rng = np.random.default_rng(0)
    n, H, dh = 50, 3, 16
    q, k, v = _qkv(rng, n, H, dh)
    causal = np.tril(np.ones((n, n), dtype=bool))
    O, _ = attention.masked_attention(q, k, v, causal, 1 / np.sqrt(dh))
    t = lambda a: torch.tensor(a, dtype=torch.float64).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", ["train", "test"])
def test_matches_scalar_loop(mode):
    rng = np.random.default_rng(1)
    n, dh = 19, 4
    starts = chunks.uniform_starts(n, 4, 1)
    q, k, v = _qkv(rng, n, 1, dh)
    M = mask.dense_mask(n, starts, 2, mode)
    O, _ = attention.masked_attention(q, k, v, M, 0.5)
    Os = scalar.attention(q[:, 0].tolist(), k[:, 0].tolist(), v[:, 0].tolist(), lambda i, j: bool(M[i, j]), 0.5)
    np.testing.assert_allclose(O[:, 0], np.array(Os), rtol=1e-12, atol=1e-13)


def test_lse_matches_library_logsumexp():
    rng = np.random.default_rng(2)
    n, H, dh = 30, 2, 8
    q, k, v = _qkv(rng, n, H, dh)
    starts = chunks.uniform_starts(n, 3, 0)
    M = mask.dense_mask(n, starts, 2, "train")
    _, lse = attention.masked_attention(q, k, v, M, 0.3)
    logits = np.einsum("ihd,jhd->hij", q, k) * 0.3
    ref = scipy.special.logsumexp(np.where(M[None], logits, -np.inf), axis=2)
    np.testing.assert_allclose(lse, ref, rtol=1e-12)


def test_softmax_invariants():
    rng = np.random.default_rng(3)
    n, H, dh = 40, 2, 8
    q, k, v = _qkv(rng, n, H, dh)
    starts = chunks.uniform_starts(n, 4, 2)
    M = mask.dense_mask(n, starts, 3, "test")
    # V == 1 gives O == 1 on every row with a key
    O1, _ = attention.masked_attention(q, k, np.ones_like(v), M, 0.4)
    np.testing.assert_allclose(O1, 1.0, rtol=1e-13)
    # permuting the keys (and the mask columns with them) changes nothing
    perm = rng.permutation(n)
    O, lse = attention.masked_attention(q, k, v, M, 0.4)
    Op, lsep = attention.masked_attention(q, k[perm], v[perm], M[:, perm], 0.4)
    np.testing.assert_allclose(Op, O, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lsep, lse, rtol=1e-12)
    # a component of q orthogonal to all keys... replaced by a constant logit shift:
    # adding c * e to every key and c' to q along e shifts each row's logits by a constant
    e = np.zeros(dh)
    e[0] = 1.0
    k2 = k.copy()
    k2[..., 0] = 0.0
    q2 = q.copy()
    q2[..., 0] = 0.0
    k3 = k2 + e
    Oa, _ = attention.masked_attention(q2, k2, v, M, 0.4)
    Ob, _ = attention.masked_attention(q2 + 5.0 * e, k3, v, M, 0.4)
    np.testing.assert_allclose(Ob, Oa, rtol=1e-12, atol=1e-13)


def test_empty_rows():
    n, dh = 12, 4
    rng = np.random.default_rng(4)
    q, k, v = _qkv(rng, n, 1, dh)
    starts = chunks.uniform_starts(n, 4, 0)
    M = mask.dense_mask(n, starts, 0, "test")
    O, lse = attention.masked_attention(q, k, v, M, 1.0)
    assert np.all(O[:3] == 0) and np.all(np.isneginf(lse[:, :3]))
    assert np.all(np.isfinite(lse[:, 3:]))


def test_rows_variant_matches_dense():
    rng = np.random.default_rng(5)
    n, H, dh = 33, 2, 8
    q, k, v = _qkv(rng, n, H, dh)
    starts = chunks.varlen_starts(rng.integers(2, 7, size=n).tolist(), n)
    M = mask.dense_mask(n, starts, 4, "train")
    O, lse = attention.masked_attention(q, k, v, M, 0.25)
    rows = [0, 5, 17, 32]
    Or, lser = attention.attention_rows(q, k, v, rows, [np.nonzero(M[i])[0] for i in rows], 0.25)
    np.testing.assert_allclose(Or, O[rows], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lser, lse[:, rows], rtol=1e-12)


def test_layer_with_chunk_size_one_is_causal_attention_over_per_token_maps():
    """P = 1 collapses the SSM to k_t = delta x_t (B_t . C_t) and the layer to causal attention."""
    rng = np.random.default_rng(6)
    n, H, dh, N = 24, 2, 4, 16
    D = H * dh
    x = rng.standard_normal((n, D))
    dts = [rng.standard_normal((n, D)) - 1 for _ in range(2)]
    bias = [rng.uniform(-4, -1, D) for _ in range(2)]
    A = [-np.exp(rng.uniform(0, np.log(16), (D, N))) for _ in range(2)]
    BC = [(rng.standard_normal((n, N)), rng.standard_normal((n, N))) for _ in range(2)]
    q = rng.standard_normal((n, H, dh))
    starts = chunks.uniform_starts(n, 1)
    is_start = chunks.is_start_mask(starts, n)
    K, _ = ssm.selective_scan(x, dts[0], bias[0], A[0], BC[0][0], BC[0][1], is_start)
    V, _ = ssm.selective_scan(x, dts[1], bias[1], A[1], BC[1][0], BC[1][1], is_start)
    M = mask.dense_mask(n, starts, 0, "train")
    O, _ = attention.masked_attention(q, K.reshape(n, H, dh), V.reshape(n, H, dh), M, 1 / np.sqrt(dh))
    kk = (ssm.softplus(dts[0] + bias[0]) * x * (BC[0][0] * BC[0][1]).sum(1)[:, None]).reshape(n, H, dh)
    vv = (ssm.softplus(dts[1] + bias[1]) * x * (BC[1][0] * BC[1][1]).sum(1)[:, None]).reshape(n, H, dh)
    t = lambda a: torch.tensor(a, dtype=torch.float64).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(kk), t(vv), is_causal=True,
                                                           scale=1 / np.sqrt(dh)).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-11, atol=1e-12)
