"""Prefill -> decode cache handoff (attamba_cache_from_prefill) on the GPU.

The cache a prefill of [0, n0) leaves is checked against the oracle's
`decode.cache_from_prefill` (boundary positions, copied rows, the SSM states
after n0 - 1 from the oracle scan), and decoding positions n0 .. n - 1 from it
must reproduce the M_test prefill rows, as decoding from an empty cache does.
"""

import numpy as np
import pytest
import torch

from helpers import BF16_ATOL, Guarded, assert_written, empty_cache_contents, f64, gpu_cache, run_prefill
from oracle import chunks as OC
from oracle import decode as OD
from oracle import ssm as OS
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P,offset,L,n0,N", [(8, 3, 16, 300, 16), (4, 0, 8, 256, 16), (8, 0, 64, 40, 16),
                                             (3, 1, 1, 100, 16), (8, 3, 16, 300, 32)])
def test_cache_from_prefill_matches_oracle_and_continues_the_prefill(P, offset, L, n0, N):
    B, H, dh, m = 2, 2, 64, 24
    n = n0 + m
    D = H * dh
    cfg = W.shrink(W.BF16_TEST_P8_L64, B=B, n=n, D=D, H=H, P=P, offset=offset, L=L, mode="test", N=N)
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)                      # M_test prefill over all n positions (reference rows)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    head = lambda t: t[:, :n0].contiguous()
    K0 = pf.K.view(B, n, H, dh)[:, :n0].contiguous()
    V0 = pf.V.view(B, n, H, dh)[:, :n0].contiguous()
    flat = lambda t: head(t).view(B * n0, -1)
    cap = n // P + 2
    guard = Guarded()
    cache = gpu_cache(empty_cache_contents(B, H, dh, N, L, cap), P, offset, guard)   # NaN until written
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.cache_from_prefill(cache, K0, V0, flat(g["x"]), flat(g["dt_k"]), flat(g["dt_v"]), g["bias_k"], g["bias_v"],
                         g["A_k"], g["A_v"], flat(g["B_k"]), flat(g["C_k"]), flat(g["B_v"]), flat(g["C_v"]), n0, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    guard.check()
    assert_written(cache.state, "state")

    # bookkeeping and copied rows against the oracle's rule
    ends = [p for p in range(n0) if OD.is_chunk_end(p, P, offset)]
    nb = len(ends)
    assert torch.all(cache.nb == nb) and torch.all(cache.pos == n0)
    assert cache.bpos[:, :nb].cpu().numpy().tolist() == [ends] * B
    for k, p in enumerate(ends):
        assert torch.equal(cache.Kb[:, :, k], K0[:, p]) and torch.equal(cache.Vb[:, :, k], V0[:, p])
    for p in range(max(0, n0 - L), n0):
        assert torch.equal(cache.Kr[:, :, p % L], K0[:, p]) and torch.equal(cache.Vr[:, :, p % L], V0[:, p])

    # SSM states after n0 - 1 against the oracle scan of [0, n0)
    starts = OC.uniform_starts(n0, P, offset)
    is_start = OC.is_start_mask(starts, n0)
    state = cache.state.cpu().numpy().astype(np.float64)       # [2, B, N, D]
    for b in range(B):
        for s, name in enumerate(("k", "v")):
            _, h = OS.selective_scan(f64(inp["x"][b, :n0]), f64(inp["dt_" + name][b, :n0]), f64(inp["bias_" + name]),
                                     f64(inp["A_" + name]), f64(inp["B_" + name][b, :n0]),
                                     f64(inp["C_" + name][b, :n0]), is_start)
            np.testing.assert_allclose(state[s, b].T, h, rtol=1e-4, atol=1e-4 * np.abs(h).max())

    # decoding n0 .. n - 1 from the handed-off cache continues the prefill
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device="cuda")
    O_pre = pf.O.view(B, n, H, dh)
    for t in range(n0, n):
        o = guard((B, H, dh), torch.bfloat16)
        c = lambda name: g[name][:, t].contiguous()
        A.decode_step(cache, c("q"), c("x"), c("dt_k"), c("dt_v"), g["bias_k"], g["bias_v"], g["A_k"], g["A_v"],
                      c("B_k"), c("C_k"), c("B_v"), c("C_v"), inp["scale"], o, ws, status)
        err = (o.float() - O_pre[:, t].float()).abs().max().item()
        assert err <= BF16_ATOL, (t, err)
    torch.cuda.synchronize()
    guard.check()
    assert status.item() == 0
