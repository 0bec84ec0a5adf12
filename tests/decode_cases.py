"""Decode runs shared by the decode tests and the no-alloc entry point's test: GPU steps into
poisoned, guarded outputs, and the oracle's decode on the same inputs."""

import numpy as np
import torch

from helpers import (Guarded, assert_bf16_close, assert_written, decode_rounding_bound, empty_cache_contents, f64,
                     gpu_cache, oracle_step, run_prefill)
from oracle import chunks as OC
from oracle import decode as OD
from oracle import ssm as OS
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import workloads as W


def step_inputs(src, s=None, col=None):
    """Device inputs of one step: per-step arrays [steps, B, ...] at s, or prefill arrays [B, n, ...]
    at position col."""
    names = ("q", "x", "dt_k", "dt_v", "B_k", "C_k", "B_v", "C_v")
    if col is None:
        return {k: src[k][s] for k in names}
    return {k: src[k][:, col].contiguous() for k in names}


def gpu_step(cache, g, si, scale, guard, status, workspace=None, noalloc=False):
    cfg_B, H, dh = cache.B, cache.H, cache.dh
    o = guard((cfg_B, H, dh), torch.bfloat16)
    args = (si["q"], si["x"], si["dt_k"], si["dt_v"], g["bias_k"], g["bias_v"], g["A_k"], g["A_v"], si["B_k"],
            si["C_k"], si["B_v"], si["C_v"], scale, o)
    if noalloc:
        A.decode_step_noalloc(cache, *args, status)
    else:
        A.decode_step(cache, *args, workspace, status)
    return o


def run_steps(dec, g, cache, steps, status, guard):
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device="cuda")
    outs = [gpu_step(cache, g, step_inputs(g, s), dec["scale"], guard, status, ws) for s in range(steps)]
    torch.cuda.synchronize()
    guard.check()
    for s, o in enumerate(outs):
        assert_written(o, f"o_t step {s}")
    return outs


def decode_from_empty_vs_oracle(cfg, steps, noalloc=False):
    """Decode ``steps`` tokens from an empty cache of the workload's capacity; every output of
    every sequence against the oracle's decode from its own empty cache."""
    dec = W.make_decode(cfg)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in dec.items()}
    contents = empty_cache_contents(cfg.B, cfg.H, cfg.dh, cfg.N, cfg.L, dec["cap"])
    guard = Guarded()
    cache = gpu_cache(contents, cfg.P, cfg.offset, guard)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = None if noalloc else torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device="cuda")
    outs = [gpu_step(cache, g, step_inputs(g, s), dec["scale"], guard, status, ws, noalloc) for s in range(steps)]
    torch.cuda.synchronize()
    guard.check()
    assert status.item() == 0
    rows = list(range(cfg.B))
    oc = OD.DecodeCache(cfg.B, cfg.H, cfg.dh, cfg.N, cfg.P, cfg.offset, cfg.L)
    for s in range(steps):
        assert_written(outs[s], f"o_t step {s}")
        ro = oracle_step(oc, dec, s, rows, dec["scale"])
        got = f64(outs[s])
        for b in rows:
            extra = decode_rounding_bound(oc, b, f64(dec["q"][s][b]), ro[b], 0, dec["scale"])
            assert_bf16_close(got[b], ro[b], f"step {s} b={b}", extra=extra)
    assert torch.all(cache.pos == steps)
    return cache


def handoff_then_decode(n0, steps, cap, noalloc=False):
    """A prefill of n0 tokens (M_test, P 8, L 64, B 1, H 2) handed into a cache of capacity ``cap``,
    then ``steps`` decode steps; against the oracle's scan, cache_from_prefill and decode.  With
    cap 2064 the step splits each key set 16 ways while the set holds about 70 keys, so most splits
    are empty and the newest key lies far from the last split's nominal range."""
    B, H, dh, N, P, offset, L = 1, 2, 64, 16, 8, 0, 64
    n = n0 + steps
    cfg = W.shrink(W.BF16_TEST_P8_L64, B=B, n=n, D=H * dh, H=H, P=P, offset=offset, L=L, mode="test", N=N,
                   seed=53)
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    head = lambda t: t[:, :n0].contiguous()
    flat = lambda t: head(t).view(B * n0, -1)
    K0 = pf.K.view(B, n, H, dh)[:, :n0].contiguous()
    V0 = pf.V.view(B, n, H, dh)[:, :n0].contiguous()
    guard = Guarded()
    cache = gpu_cache(empty_cache_contents(B, H, dh, N, L, cap), P, offset, guard)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.cache_from_prefill(cache, K0, V0, flat(g["x"]), flat(g["dt_k"]), flat(g["dt_v"]), g["bias_k"], g["bias_v"],
                         g["A_k"], g["A_v"], flat(g["B_k"]), flat(g["C_k"]), flat(g["B_v"]), flat(g["C_v"]), n0, status)
    ws = None if noalloc else torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device="cuda")
    outs = [gpu_step(cache, g, step_inputs(g, col=t), inp["scale"], guard, status, ws, noalloc) for t in range(n0, n)]
    torch.cuda.synchronize()
    guard.check()
    assert status.item() == 0

    # the oracle: its own scan of [0, n0), its own handoff, its own decode
    starts = OC.uniform_starts(n0, P, offset)
    is_start = OC.is_start_mask(starts, n0)
    Ks, Vs, hs = [], [], []
    for s in ("k", "v"):
        y, h = OS.selective_scan(f64(inp["x"][0, :n0]), f64(inp["dt_" + s][0, :n0]), f64(inp["bias_" + s]),
                                 f64(inp["A_" + s]), f64(inp["B_" + s][0, :n0]), f64(inp["C_" + s][0, :n0]), is_start)
        (Ks if s == "k" else Vs).append(y.reshape(n0, H, dh))
        hs.append(h)
    oc = OD.cache_from_prefill(np.stack(Ks), np.stack(Vs), np.stack(hs)[:, None], n0, P, offset, L, H, dh, N)
    for k, t in enumerate(range(n0, n)):
        assert_written(outs[k], f"o_t position {t}")
        ro = oracle_step(oc, inp, None, [0], inp["scale"], col=t)
        extra = decode_rounding_bound(oc, 0, f64(inp["q"][0, t]), ro[0], 0, inp["scale"])
        assert_bf16_close(f64(outs[k][0]), ro[0], f"position {t}", extra=extra)
    return cache
