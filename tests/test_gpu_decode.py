"""GPU decode step vs the oracle: the 128-step workload on its synthetic cache, decode from an
empty cache (small, and at the workload's dimensions and capacity), decode after a short prefill
handed into a long-capacity cache, decode from an empty cache against the M_test prefill rows, and
the full-cache status bit.

Every cache array and every o_t lives in a poisoned buffer with a guard region (helpers.Guarded):
cache rows not yet written hold NaN, so a step that reads past the boundary count or a ring slot
it did not fill gives NaN, and a write past an array's end changes its guard.
"""

import numpy as np
import pytest
import torch

from decode_cases import decode_from_empty_vs_oracle, gpu_step, handoff_then_decode, run_steps, step_inputs
from helpers import (BF16_ATOL, Guarded, assert_bf16_close, assert_written, decode_cache_contents,
                     decode_rounding_bound, empty_cache_contents, f64, gpu_cache, oracle_cache, oracle_step,
                     run_prefill)
from oracle import decode as OD
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_decode_workload_128_steps():
    cfg = W.DECODE_CONFIG
    dec = W.make_decode(cfg)
    contents = decode_cache_contents(dec)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in dec.items()}
    guard = Guarded()
    cache = gpu_cache(contents, cfg.P, cfg.offset, guard)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = run_steps(dec, g, cache, cfg.steps, status, guard)
    assert status.item() == 0
    rows = [0, cfg.B - 1]
    oc = oracle_cache(contents, cfg, rows)
    for s in range(cfg.steps):
        ro = oracle_step(oc, dec, s, rows, dec["scale"])
        for r, b in enumerate(rows):
            extra = decode_rounding_bound(oc, r, f64(dec["q"][s][b]), ro[r], cfg.ctx, dec["scale"])
            assert_bf16_close(f64(outs[s][b]), ro[r], f"step {s} b={b}", extra=extra)
    # cache bookkeeping: positions advanced, one boundary appended per completed chunk
    end = cfg.ctx + cfg.steps
    ends = [p for p in range(end) if OD.is_chunk_end(p, cfg.P, cfg.offset)]
    assert torch.all(cache.pos == end)
    assert torch.all(cache.nb == len(ends))
    assert cache.bpos[0, : len(ends)].cpu().tolist() == ends
    # appended boundary keys equal the ring entries written at the same positions
    last = len(ends) - 1
    p = ends[last]
    if p > end - 1 - cfg.L:
        assert torch.equal(cache.Kb[:, :, last], cache.Kr[:, :, p % cfg.L])


@pytest.mark.parametrize("ctx,L,offset", [(16384, 64, 0), (5000, 40, 5)])
def test_decode_many_splits(ctx, L, offset):
    """Few (sequence, head) pairs over a long context: the step splits each key set many ways (16 at
    ctx 16384), so splits start and end inside stages, one stage mixes boundary rows with ring rows
    before and after the ring's wrap, and the last split holds the newest key."""
    cfg = W.shrink(W.DECODE_CONFIG, B=1, H=2, D=128, ctx=ctx, L=L, offset=offset, steps=24, seed=31)
    dec = W.make_decode(cfg)
    contents = decode_cache_contents(dec)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in dec.items()}
    guard = Guarded()
    cache = gpu_cache(contents, cfg.P, cfg.offset, guard)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = run_steps(dec, g, cache, cfg.steps, status, guard)
    assert status.item() == 0
    oc = oracle_cache(contents, cfg, [0])
    for s in range(cfg.steps):
        ro = oracle_step(oc, dec, s, [0], dec["scale"])
        extra = decode_rounding_bound(oc, 0, f64(dec["q"][s][0]), ro[0], ctx, dec["scale"])
        assert_bf16_close(f64(outs[s][0]), ro[0], f"step {s}", extra=extra)
    assert torch.all(cache.pos == ctx + cfg.steps)


def test_decode_from_empty_cache_at_workload_size():
    """The decode workload's dimensions and capacity (B 32, H 32, cap 2066: two splits per sequence and
    head) starting from an empty cache: at t = 0 the key set is one key, so one split has none.  The
    split that runs the SSM step must be the one holding the newest key (pith.science review, "Core
    claim": the boundary-state cache grows chunk by chunk from an empty context)."""
    cfg = W.shrink(W.DECODE_CONFIG, seed=41)
    cache = decode_from_empty_vs_oracle(cfg, 24)
    assert A.decode_workspace_size(cache) > 0


def test_decode_after_short_handoff_into_long_capacity():
    """B 1, H 2, cap 2064, L 64 after a prefill of 100 tokens: 16 splits over 68 keys at t = 100."""
    cache = handoff_then_decode(100, 24, 2064)
    assert A.decode_workspace_size(cache) > 0


@pytest.mark.parametrize("P,offset,L,N", [(4, 0, 3, 16), (8, 3, 8, 16), (3, 1, 1, 16), (8, 3, 8, 32)])
def test_decode_from_empty_cache_equals_test_mask_prefill(P, offset, L, N):
    """Decoding n tokens one by one from an empty cache reproduces the M_test prefill rows of the GPU,
    and the oracle's own decode from an empty cache."""
    B, n, H, dh = 2, 150, 2, 64
    cfg = W.shrink(W.BF16_TEST_P8_L64, B=B, n=n, D=H * dh, H=H, P=P, offset=offset, L=L, mode="test", N=N)
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    cap = n // P + 2
    guard = Guarded()
    cache = gpu_cache(empty_cache_contents(B, H, dh, N, L, cap), P, offset, guard)
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    O_pre = pf.O.view(B, n, H, dh)
    oc = OD.DecodeCache(B, H, dh, N, P, offset, L)
    rows = list(range(B))
    for t in range(n):
        o = gpu_step(cache, g, step_inputs(g, col=t), inp["scale"], guard, status, ws)
        torch.cuda.synchronize()
        assert_written(o, f"o_t position {t}")
        err = (o.float() - O_pre[:, t].float()).abs().max().item()
        assert err <= BF16_ATOL, (t, err)
        ro = oracle_step(oc, inp, None, rows, inp["scale"], col=t)
        got = f64(o)
        for b in rows:
            extra = decode_rounding_bound(oc, b, f64(inp["q"][b, t]), ro[b], 0, inp["scale"])
            assert_bf16_close(got[b], ro[b], f"position {t} b={b}", extra=extra)
    guard.check()
    assert status.item() == 0


def test_full_cache_raises_status_bit():
    B, H, dh, N, P, L, cap = 1, 1, 64, 16, 2, 2, 3
    dev = "cuda"
    guard = Guarded()
    contents = empty_cache_contents(B, H, dh, N, L, cap)
    cache = gpu_cache(contents, P, 0, guard)
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device=dev)
    f = lambda *s: torch.zeros(*s, dtype=torch.float32, device=dev)
    for _ in range(2 * cap + 2):
        A.decode_step(cache, z(B, H, dh), z(B, H * dh), z(B, H * dh), z(B, H * dh), f(H * dh), f(H * dh),
                      -torch.ones(H * dh, N, device=dev), -torch.ones(H * dh, N, device=dev), z(B, N), z(B, N),
                      z(B, N), z(B, N), 0.125, z(B, H, dh), ws, status)
    torch.cuda.synchronize()
    guard.check()
    assert status.item() & A.DEV_CACHE_FULL
    assert cache.nb.item() == cap
