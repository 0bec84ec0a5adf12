"""GPU KV-SSM scan vs the oracle's per-token recurrence."""

import numpy as np
import pytest
import torch

from helpers import Guarded, assert_close, assert_written, chunk_starts, f64, oracle_scan_seq, run_prefill
from oracle import chunks as OC
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu

SMALL = [
    W.TINY_F32_TRAIN,                                                   # fp32, full size
    W.shrink(W.BF16_TRAIN_CYCLIC, B=2, n=300, D=128, H=2),                 # cyclic offset 3, ragged n
    W.shrink(W.BF16_TEST_P8_L64, B=2, n=333, D=192, H=3),                 # P = 8
    W.shrink(W.BF16_VARLEN_TRAIN, B=3, n=257, D=128, H=2),                 # variable chunks
    W.shrink(W.BF16_TRAIN_CYCLIC, B=1, n=64, D=64, H=1, P=1, offset=0),   # P = 1
    W.shrink(W.BF16_TRAIN_CYCLIC, B=2, n=50, D=64, H=1, P=64, offset=0),  # one chunk per sequence
    W.shrink(W.TINY_F32_TRAIN, B=2, n=77, D=64, H=1, P=16, offset=5),   # fp32 cyclic
    W.shrink(W.BF16_TEST_P8_L64, B=2, n=200, D=128, H=2, N=32),           # state size 32 (the pages' default)
    W.shrink(W.BF16_VARLEN_TRAIN, B=2, n=150, D=64, H=1, N=32),            # N = 32, variable chunks
    W.shrink(W.TINY_F32_TRAIN, B=1, n=96, D=64, H=1, N=32, offset=2),   # fp32, N = 32
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"{c.name}-B{c.B}-n{c.n}-D{c.D}-P{c.P}-N{c.N}")
def test_scan_small(cfg):
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    K = pf.K.view(cfg.B, cfg.n, cfg.D)
    V = pf.V.view(cfg.B, cfg.n, cfg.D)
    for b in range(cfg.B):
        rk, rv = oracle_scan_seq(inp, b)
        assert_close(cfg.dtype, f64(K[b]), rk, f"K b={b}")
        assert_close(cfg.dtype, f64(V[b]), rv, f"V b={b}")
    # chunk-end rows are the same values as the full outputs at the chunk ends (bit-exact copy)
    ends = np.array([b * cfg.n + e for b, st in enumerate(chunk_starts(inp)) for e in OC.boundary_positions(st, cfg.n)])
    assert torch.equal(pf.Kc, pf.K[torch.from_numpy(ends).cuda()])
    assert torch.equal(pf.Vc, pf.V[torch.from_numpy(ends).cuda()])
    assert pf.status.item() == 0


@pytest.mark.parametrize("cfg", [W.BF16_TRAIN_CYCLIC, W.BF16_TEST_P8_L64, W.BF16_VARLEN_TRAIN], ids=lambda c: c.name)
def test_scan_full_size_sampled_chunks(cfg):
    """The workloads at full size, in the launch the bench times; the oracle recomputes sampled chunks."""
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    K = pf.K.view(cfg.B, cfg.n, cfg.D)
    V = pf.V.view(cfg.B, cfg.n, cfg.D)
    rng = np.random.default_rng(cfg.seed)
    for b in (0, cfg.B - 1):
        st = list(chunk_starts(inp)[b]) + [cfg.n]
        picks = {0, len(st) - 2} | set(rng.integers(0, len(st) - 1, size=4).tolist())
        for c in sorted(picks):
            t0, t1 = st[c], st[c + 1]
            rk, rv = oracle_scan_seq(inp, b, t0, t1)
            assert_close(cfg.dtype, f64(K[b, t0:t1]), rk, f"K b={b} chunk={c}")
            assert_close(cfg.dtype, f64(V[b, t0:t1]), rv, f"V b={b} chunk={c}")
    assert pf.status.item() == 0


@pytest.mark.parametrize("cfg", [W.shrink(W.BF16_TRAIN_CYCLIC, B=2, n=300, D=128, H=2),
                                 W.shrink(W.TINY_F32_TRAIN, B=2, n=77, D=64, H=1, P=16, offset=5)],
                         ids=lambda c: f"{c.name}-n{c.n}-D{c.D}")
def test_scan_kept_projection_inputs(cfg):
    """attamba_kv_ssm_scan_u: the keys SSM reads u_k = x W_K, the values SSM u_v = x W_V (the
    kept-projection variant); each must match the oracle recurrence over its own input, and u_k = u_v = x
    must reproduce attamba_kv_ssm_scan bit for bit."""
    from ssm_compressed_chunked_b200 import attamba as A, layer
    from oracle import ssm as OS
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    gen = torch.Generator().manual_seed(11)
    dt = W.torch_dtype(cfg.dtype)
    proj = [torch.randn(cfg.D, cfg.D, generator=gen) / cfg.D ** 0.5 for _ in range(2)]
    x32 = inp["x"].float().reshape(-1, cfg.D)
    u = [(x32 @ w).to(dt) for w in proj]                     # the caller's projections, rounded like q
    T = cfg.B * cfg.n
    guard = Guarded()
    K = guard((T, cfg.D), dt)
    V = guard((T, cfg.D), dt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flat = lambda t: t.reshape(T, -1)
    args = (flat(g["dt_k"]), flat(g["dt_v"]), g["bias_k"], g["bias_v"], g["A_k"], g["A_v"], flat(g["B_k"]),
            flat(g["C_k"]), flat(g["B_v"]), flat(g["C_v"]), pf.index.cu, pf.n_chunks)
    A.kv_ssm_scan_u(u[0].cuda(), u[1].cuda(), *args, K, V, status=status)
    # shared input through the new entry point equals the original one exactly
    K2 = guard((T, cfg.D), dt)
    V2 = guard((T, cfg.D), dt)
    A.kv_ssm_scan_u(flat(g["x"]), flat(g["x"]), *args, K2, V2, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    guard.check()
    for name, t in (("K", K), ("V", V), ("K2", K2), ("V2", V2)):
        assert_written(t, name)
    assert torch.equal(K2, pf.K) and torch.equal(V2, pf.V)
    for b in range(cfg.B):
        is_start = OC.is_start_mask(np.asarray(chunk_starts(inp)[b]), cfg.n)
        sl = slice(b * cfg.n, (b + 1) * cfg.n)
        for s, name, out in ((0, "k", K), (1, "v", V)):
            ref, _ = OS.selective_scan(f64(u[s][sl]), f64(inp["dt_" + name][b]), f64(inp["bias_" + name]),
                                       f64(inp["A_" + name]), f64(inp["B_" + name][b]), f64(inp["C_" + name][b]),
                                       is_start)
            assert_close(cfg.dtype, f64(out[sl]), ref, f"{name} b={b}")


@pytest.mark.parametrize("dtype_cfg", [W.shrink(W.TINY_F32_TRAIN, B=1, n=96, D=64, H=1, P=8, offset=0),
                                       W.shrink(W.BF16_TEST_P8_L64, B=1, n=96, D=64, H=1)],
                         ids=["f32", "bf16"])
def test_scan_softplus_regimes(dtype_cfg):
    """dt spread over [-120, 40] so softplus(dt + bias) meets each regime of the kernel's evaluation:
    the linear one above 20, the logarithm of 1 + e^z around 0, the series for small e^z, and steps
    whose e^z underflows in fp32 (no decay and no input at all)."""
    cfg = dtype_cfg
    inp = W.make_layer(cfg)
    gen = torch.Generator().manual_seed(77)
    for k in ("dt_k", "dt_v"):
        z = (torch.rand(inp[k].shape, generator=gen) * 160.0 - 120.0)
        inp[k] = z.to(inp[k].dtype)
    pf = run_prefill(inp, cfg)
    K = pf.K.view(cfg.B, cfg.n, cfg.D)
    V = pf.V.view(cfg.B, cfg.n, cfg.D)
    rk, rv = oracle_scan_seq(inp, 0)
    assert_close(cfg.dtype, f64(K[0]), rk, "K")
    assert_close(cfg.dtype, f64(V[0]), rv, "V")
    assert pf.status.item() == 0
