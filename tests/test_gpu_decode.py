"""GPU decode step vs the oracle: the 128-step workload on its synthetic cache,
decode from an empty cache against the M_test prefill rows, and the full-cache status bit."""

import numpy as np
import pytest
import torch

from helpers import BF16_ATOL, BF16_HALF_ULP, assert_bf16_close, f64, run_prefill
from oracle import decode as OD
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu


def gpu_cache(dec, B=None):
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in dec.items()}
    cfg = dec["cfg"]
    return g, A.Cache(g["state"].clone(), g["Kb"].clone(), g["Vb"].clone(), g["bpos"].clone(), g["Kr"].clone(),
                      g["Vr"].clone(), g["nbuf"].clone(), g["pos"].clone(), cfg.P, cfg.offset)


def oracle_cache(dec, rows):
    """The same synthetic cache in the oracle's format, for the batch rows `rows`."""
    cfg = dec["cfg"]
    c = OD.DecodeCache(len(rows), cfg.H, cfg.dh, cfg.N, cfg.P, cfg.offset, cfg.L)
    c.state = np.transpose(f64(dec["state"][:, rows]), (0, 1, 3, 2)).copy()
    nb = dec["nb"]
    for r, b in enumerate(rows):
        c.bpos[r] = dec["bpos"][b, :nb].tolist()
        Kb = f64(dec["Kb"][b, :, :nb])
        Vb = f64(dec["Vb"][b, :, :nb])
        c.Kb[r] = [Kb[:, k] for k in range(nb)]
        c.Vb[r] = [Vb[:, k] for k in range(nb)]
        for p in range(cfg.ctx - cfg.L, cfg.ctx):
            c.ring[r][p] = (f64(dec["Kr"][b, :, p % cfg.L]), f64(dec["Vr"][b, :, p % cfg.L]))
        c.pos[r] = cfg.ctx
    return c


def run_steps(dec, g, cache, steps, status):
    cfg = dec["cfg"]
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device="cuda")
    outs = []
    for s in range(steps):
        o = torch.empty(cfg.B, cfg.H, cfg.dh, dtype=torch.bfloat16, device="cuda")
        A.decode_step(cache, g["q"][s], g["x"][s], g["dt_k"][s], g["dt_v"][s], g["bias_k"], g["bias_v"],
                      g["A_k"], g["A_v"], g["B_k"][s], g["C_k"][s], g["B_v"][s], g["C_v"][s], dec["scale"], o, ws,
                      status)
        outs.append(o)
    torch.cuda.synchronize()
    return outs


def test_decode_workload_128_steps():
    cfg = W.DECODE_CONFIG
    dec = W.make_decode(cfg)
    g, cache = gpu_cache(dec)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = run_steps(dec, g, cache, cfg.steps, status)
    assert status.item() == 0
    rows = [0, cfg.B - 1]
    oc = oracle_cache(dec, rows)
    worst = 0.0
    for s in range(cfg.steps):
        sel = lambda t: f64(t[s][rows])
        ro = oc.step(sel(dec["q"]), sel(dec["x"]), np.stack([f64(dec["dt_k"][s][rows]), f64(dec["dt_v"][s][rows])]),
                     np.stack([f64(dec["bias_k"]), f64(dec["bias_v"])]), np.stack([f64(dec["A_k"]), f64(dec["A_v"])]),
                     np.stack([f64(dec["B_k"][s][rows]), f64(dec["B_v"][s][rows])]),
                     np.stack([f64(dec["C_k"][s][rows]), f64(dec["C_v"][s][rows])]), dec["scale"])
        err = np.abs(f64(outs[s][rows]) - ro).max()
        worst = max(worst, err)
        assert err <= BF16_ATOL, (s, err)
    # cache bookkeeping: positions advanced, one boundary appended per completed chunk
    end = cfg.ctx + cfg.steps
    exp_nb = sum(1 for p in range(end) if OD.is_chunk_end(p, cfg.P, cfg.offset))
    assert torch.all(cache.pos == end)
    assert torch.all(cache.nb == exp_nb)
    assert cache.bpos[0, exp_nb - 1].item() == max(p for p in range(end) if OD.is_chunk_end(p, cfg.P, cfg.offset))
    # appended boundary keys equal the ring entries written at the same positions
    last = exp_nb - 1
    p = cache.bpos[0, last].item()
    if p > end - 1 - cfg.L:
        assert torch.equal(cache.Kb[:, :, last], cache.Kr[:, :, p % cfg.L])


def decode_rounding_bound(oc, b, q, o_ref, ctx, scale):
    """First-order effect on the output of keys the GPU stored in bf16 while the oracle keeps them in
    float64: the keys and values written during the decode (positions >= ctx; the synthetic cache
    itself is bf16 on both sides).  Same rule as the prefill attention's: a change dv moves o by at most
    max |dv|, a change dk moves a score by at most scale sum |q| |dk| and o by at most
    max |v - o| times that.  Returns [H, dh]."""
    t = oc.pos[b] - 1
    lo = max(0, t - oc.L + 1)
    ks, vs = [], []
    for p, kk, vv in zip(oc.bpos[b], oc.Kb[b], oc.Vb[b]):
        if ctx <= p < lo:
            ks.append(kk)
            vs.append(vv)
    for p in range(max(lo, ctx), t + 1):
        kk, vv = oc.ring[b][p]
        ks.append(kk)
        vs.append(vv)
    if not ks:
        return np.zeros_like(o_ref)
    k = np.stack(ks)                                               # [j, H, dh]
    v = np.stack(vs)
    ds = scale * BF16_HALF_ULP * np.einsum("hd,jhd->jh", np.abs(q), np.abs(k)).max(axis=0)    # [H]
    dv = BF16_HALF_ULP * np.abs(v).max(axis=0)                                                 # [H, dh]
    spread = np.abs(v - o_ref[None]).max(axis=0)
    return dv + spread * ds[:, None]


@pytest.mark.parametrize("ctx,L,offset", [(16384, 64, 0), (5000, 40, 5)])
def test_decode_many_splits(ctx, L, offset):
    """Few (sequence, head) pairs over a long context: the step splits each key set many ways (16 at
    ctx 16384), so splits start and end inside stages, one stage mixes boundary rows with ring rows
    before and after the ring's wrap, and the last split holds the newest key."""
    cfg = W.shrink(W.DECODE_CONFIG, B=1, H=2, D=128, ctx=ctx, L=L, offset=offset, steps=24, seed=31)
    dec = W.make_decode(cfg)
    g, cache = gpu_cache(dec)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = run_steps(dec, g, cache, cfg.steps, status)
    assert status.item() == 0
    rows = [0]
    oc = oracle_cache(dec, rows)
    for s in range(cfg.steps):
        sel = lambda t: f64(t[s][rows])
        ro = oc.step(sel(dec["q"]), sel(dec["x"]), np.stack([f64(dec["dt_k"][s][rows]), f64(dec["dt_v"][s][rows])]),
                     np.stack([f64(dec["bias_k"]), f64(dec["bias_v"])]), np.stack([f64(dec["A_k"]), f64(dec["A_v"])]),
                     np.stack([f64(dec["B_k"][s][rows]), f64(dec["B_v"][s][rows])]),
                     np.stack([f64(dec["C_k"][s][rows]), f64(dec["C_v"][s][rows])]), dec["scale"])
        extra = decode_rounding_bound(oc, 0, f64(dec["q"][s][0]), ro[0], ctx, dec["scale"])
        assert_bf16_close(f64(outs[s][rows])[0], ro[0], f"step {s}", extra=extra)
    assert torch.all(cache.pos == ctx + cfg.steps)


@pytest.mark.parametrize("P,offset,L,N", [(4, 0, 3, 16), (8, 3, 8, 16), (3, 1, 1, 16), (8, 3, 8, 32)])
def test_decode_from_empty_cache_equals_test_mask_prefill(P, offset, L, N):
    """Decoding n tokens one by one from an empty cache reproduces the M_test prefill (GPU vs GPU and vs oracle)."""
    B, n, H, dh = 2, 150, 2, 64
    cfg = W.shrink(W.BF16_TEST_P8_L64, B=B, n=n, D=H * dh, H=H, P=P, offset=offset, L=L, mode="test", N=N)
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    cap = n // P + 2
    dev = "cuda"
    cache = A.Cache(torch.zeros(2, B, N, H * dh, device=dev), torch.zeros(B, H, cap, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, H, cap, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, cap, dtype=torch.int32, device=dev),
                    torch.zeros(B, H, L, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, H, L, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, dtype=torch.int32, device=dev), torch.zeros(B, dtype=torch.int32, device=dev),
                    P, offset)
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    O_pre = pf.O.view(B, n, H, dh)
    for t in range(n):
        o = torch.empty(B, H, dh, dtype=torch.bfloat16, device=dev)
        A.decode_step(cache, g["q"][:, t].contiguous(), g["x"][:, t].contiguous(), g["dt_k"][:, t].contiguous(),
                      g["dt_v"][:, t].contiguous(), g["bias_k"], g["bias_v"], g["A_k"], g["A_v"],
                      g["B_k"][:, t].contiguous(), g["C_k"][:, t].contiguous(), g["B_v"][:, t].contiguous(),
                      g["C_v"][:, t].contiguous(), inp["scale"], o, ws, status)
        err = (o.float() - O_pre[:, t].float()).abs().max().item()
        assert err <= BF16_ATOL, (t, err)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_full_cache_raises_status_bit():
    B, H, dh, N, P, L, cap = 1, 1, 64, 16, 2, 2, 3
    dev = "cuda"
    cache = A.Cache(torch.zeros(2, B, N, H * dh, device=dev), torch.zeros(B, H, cap, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, H, cap, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, cap, dtype=torch.int32, device=dev),
                    torch.zeros(B, H, L, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, H, L, dh, dtype=torch.bfloat16, device=dev),
                    torch.zeros(B, dtype=torch.int32, device=dev), torch.zeros(B, dtype=torch.int32, device=dev), P, 0)
    ws = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device=dev)
    f = lambda *s: torch.zeros(*s, dtype=torch.float32, device=dev)
    for _ in range(2 * cap + 2):
        A.decode_step(cache, z(B, H, dh), z(B, H * dh), z(B, H * dh), z(B, H * dh), f(H * dh), f(H * dh),
                      -torch.ones(H * dh, N, device=dev), -torch.ones(H * dh, N, device=dev), z(B, N), z(B, N),
                      z(B, N), z(B, N), 0.125, z(B, H, dh), ws, status)
    torch.cuda.synchronize()
    assert status.item() & A.DEV_CACHE_FULL
    assert cache.nb.item() == cap
