"""The projection GEMM (attamba_proj_gemm) against the oracle's float64 product."""

import numpy as np
import pytest
import torch

from helpers import f64
from oracle import projection as OP
from ssm_compressed_chunked_b200 import attamba as A

pytestmark = pytest.mark.gpu


def _check(Y, ref, X, W, what):
    """bf16 rounding of the result (half an ulp, 2^-9 relative) plus the fp32 accumulation
    error bound of a K-term dot product, sum |x||w| K 2^-24."""
    mag = np.abs(f64(X)) @ np.abs(f64(W)).T
    bound = 2.0 ** -8 * np.abs(ref) + X.shape[1] * 2.0 ** -24 * mag + 1e-6
    err = np.abs(f64(Y) - ref)
    k = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"{what}: err {err[k]:.3e} > bound {bound[k]:.3e} at {k}"


@pytest.mark.parametrize("M,K,widths", [(300, 128, [64, 64, 8, 8]),            # ragged rows, one N tile
                                        (512, 1024, [1024, 1024, 1024, 16, 16, 16, 16]),  # a layer's inputs
                                        (129, 64, [72]),                          # Nout below a tile
                                        (257, 256, [256, 512])])                  # several N tiles
def test_proj_gemm_matches_oracle(M, K, widths):
    gen = torch.Generator().manual_seed(M + K)
    Nout = sum(widths)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    W = (torch.randn(Nout, K, generator=gen) / K ** 0.5).to(torch.bfloat16)
    outs, c = [], 0
    for w in widths:
        outs.append((torch.full((M, w), float("nan"), dtype=torch.bfloat16, device="cuda"), c))
        c += w
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.proj_gemm(X.cuda(), W.cuda(), outs, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = OP.split(OP.project(f64(X), f64(W)), widths)
    for k, ((t, _), r) in enumerate(zip(outs, ref)):
        _check(t.cpu(), r, X, W[sum(widths[:k]):sum(widths[:k + 1])], f"segment {k}")


def test_proj_gemm_skips_columns_no_segment_names():
    M, K, Nout = 128, 128, 96
    gen = torch.Generator().manual_seed(5)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16).cuda()
    W = torch.randn(Nout, K, generator=gen).to(torch.bfloat16).cuda()
    a = torch.zeros(M, 16, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(M, 8, dtype=torch.bfloat16, device="cuda")
    A.proj_gemm(X, W, [(a, 8), (b, 64)])
    ref = OP.project(f64(X.cpu()), f64(W.cpu()))
    _check(a.cpu(), ref[:, 8:24], X.cpu(), W.cpu()[8:24], "a")
    _check(b.cpu(), ref[:, 64:72], X.cpu(), W.cpu()[64:72], "b")


def test_proj_gemm_more_tiles_than_resident_pairs():
    """320 output tiles of 256 x 256 against 74 resident CTA pairs: every pair runs several tiles, so
    both TMEM accumulators are reused and the stage ring wraps many times."""
    M, K, widths = 8192, 128, [1024, 1024, 512]
    gen = torch.Generator().manual_seed(11)
    Nout = sum(widths)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    W = (torch.randn(Nout, K, generator=gen) / K ** 0.5).to(torch.bfloat16)
    outs, c = [], 0
    for w in widths:
        outs.append((torch.full((M, w), float("nan"), dtype=torch.bfloat16, device="cuda"), c))
        c += w
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.proj_gemm(X.cuda(), W.cuda(), outs, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = OP.split(OP.project(f64(X), f64(W)), widths)
    for k, ((t, _), r) in enumerate(zip(outs, ref)):
        _check(t.cpu(), r, X, W[sum(widths[:k]):sum(widths[:k + 1])], f"segment {k}")


@pytest.mark.parametrize("widths", [[1024, 1024, 1024, 16, 16, 16, 16], [1024]], ids=["inputs", "output"])
def test_proj_gemm_layer_size_sampled_rows(widths):
    """The layer's projections at the bench size (M = 4 x 4096 tokens, K = 1024): the seven input
    segments (q, dt_K, dt_V, B_K, C_K, B_V, C_V) and the output projection O W_O.  Every element is
    written (the outputs start as NaN); 96 sampled rows match the oracle's float64 product."""
    M, K = 16384, 1024
    gen = torch.Generator().manual_seed(12 + len(widths))
    Nout = sum(widths)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    W = (torch.randn(Nout, K, generator=gen) / K ** 0.5).to(torch.bfloat16)
    outs, c = [], 0
    for w in widths:
        outs.append((torch.full((M, w), float("nan"), dtype=torch.bfloat16, device="cuda"), c))
        c += w
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.proj_gemm(X.cuda(), W.cuda(), outs, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for k, (t, _) in enumerate(outs):
        assert not torch.isnan(t).any().item(), f"segment {k} has unwritten elements"
    rows = torch.randperm(M, generator=gen)[:96].sort().values
    Xs = X[rows]
    ref = OP.split(OP.project(f64(Xs), f64(W)), widths)
    for k, ((t, _), r) in enumerate(zip(outs, ref)):
        _check(t.cpu()[rows], r, Xs, W[sum(widths[:k]):sum(widths[:k + 1])], f"segment {k}")
