"""GPU chunk-masked attention vs the oracle's dense masked softmax.

Two levels: stage-isolated (the oracle attends over the GPU's own K/V, so the
attention error is measured alone) and end to end (the oracle also runs the
scan).  Cases span several 128-query tiles, ragged tails, tiny sequences, both
masks, the empty-row case (M_test, L = 0), L >= n, P = 1 and variable chunks.
"""

import numpy as np
import pytest
import torch

from helpers import (assert_close, assert_written, attn_rounding_bound, chunk_starts, f64, key_lists,
                     oracle_attention_seq, oracle_scan_seq, poison_, run_prefill)
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu

C1, C2, C3 = W.BF16_TRAIN_CYCLIC, W.BF16_TEST_P8_L64, W.BF16_VARLEN_TRAIN
SMALL = [
    W.TINY_F32_TRAIN,                                                    # fp32, full size
    W.shrink(W.TINY_F32_TRAIN, B=2, n=200, P=8, offset=3, L=5, mode="test"),   # fp32 M_test
    W.shrink(C1, B=2, n=300, D=128, H=2),                                  # M_train, offset 3, L 4, ragged
    W.shrink(C2, B=2, n=520, D=128, H=2),                                  # M_test P 8 L 64, 5 tiles
    W.shrink(C3, B=2, n=387, D=128, H=2),                                  # variable chunks
    W.shrink(C2, B=1, n=90, D=64, H=1),                                    # shorter than one tile
    W.shrink(C2, B=2, n=260, D=64, H=1, L=0),                              # M_test, L = 0: empty rows
    W.shrink(C1, B=1, n=200, D=64, H=1, L=500),                            # L >= n: causal
    W.shrink(C1, B=1, n=256, D=128, H=2, P=1, offset=0, L=0),              # P = 1: causal
    W.shrink(C2, B=2, n=384, D=128, H=2, P=64, L=3),                       # long chunks, M_test
    W.shrink(C1, B=1, n=300, D=64, H=1, P=128, offset=17, L=0),            # long chunks, M_train
]


def _ids(c):
    return f"{c.dtype}-{c.mode}-B{c.B}-n{c.n}-H{c.H}-P{c.P}-o{c.offset}-L{c.L}-{'var' if c.varlen else 'uni'}"


@pytest.mark.parametrize("cfg", SMALL, ids=_ids)
def test_attention_small(cfg):
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    n, H, dh = cfg.n, cfg.H, cfg.dh
    O = pf.O.view(cfg.B, n, H, dh)
    lse = pf.lse.cpu().numpy()
    K = pf.K.view(cfg.B, n, H, dh)
    V = pf.V.view(cfg.B, n, H, dh)
    starts = chunk_starts(inp)
    for b in range(cfg.B):
        st = np.asarray(starts[b])
        q = f64(inp["q"][b])
        # stage-isolated: oracle attention over the GPU's own K/V
        ro, rl = oracle_attention_seq(q, f64(K[b]), f64(V[b]), st, n, cfg.L, cfg.mode, inp["scale"])
        assert_close(cfg.dtype, f64(O[b]), ro, f"O (isolated) b={b}")
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(lse[b]), fin)
        assert_close(cfg.dtype, lse[b][fin], rl[fin], f"lse b={b}")
        # end to end: oracle scan + oracle attention
        rk, rv = oracle_scan_seq(inp, b)
        rk, rv = rk.reshape(n, H, dh), rv.reshape(n, H, dh)
        eo, _ = oracle_attention_seq(q, rk, rv, st, n, cfg.L, cfg.mode, inp["scale"])
        extra = 0.0 if cfg.dtype == "f32" else attn_rounding_bound(
            q, rk, rv, eo, key_lists(n, st, cfg.L, cfg.mode, range(n)), inp["scale"])
        assert_close(cfg.dtype, f64(O[b]), eo, f"O (end to end) b={b}", extra=extra)
    assert pf.status.item() == 0


@pytest.mark.parametrize("qscale", [6.0, 40.0])
def test_attention_wide_score_range(qscale):
    """q scaled up so a row's scores spread over tens (6x) to hundreds (40x) of units of log2: later
    tiles often hold a score far above the row's reference, so the kernel's row sum passes 2^16 or
    overflows and it moves the reference, recomputes P and rescales O (stage-isolated check)."""
    cfg = W.shrink(C2, B=2, n=520, D=128, H=2)
    inp = W.make_layer(cfg)
    inp["q"] = (inp["q"].float() * qscale).to(inp["q"].dtype)
    pf = run_prefill(inp, cfg)
    n, H, dh = cfg.n, cfg.H, cfg.dh
    O = pf.O.view(cfg.B, n, H, dh)
    lse = pf.lse.cpu().numpy()
    K = pf.K.view(cfg.B, n, H, dh)
    V = pf.V.view(cfg.B, n, H, dh)
    starts = chunk_starts(inp)
    for b in range(cfg.B):
        st = np.asarray(starts[b])
        ro, rl = oracle_attention_seq(f64(inp["q"][b]), f64(K[b]), f64(V[b]), st, n, cfg.L, cfg.mode, inp["scale"])
        assert_close(cfg.dtype, f64(O[b]), ro, f"O (q x {qscale}) b={b}")
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(lse[b]), fin)
        assert_close(cfg.dtype, lse[b][fin], rl[fin], f"lse (q x {qscale}) b={b}")
    assert pf.status.item() == 0


@pytest.mark.parametrize("cfg", [C1, C2, C3], ids=lambda c: c.name)
def test_attention_full_size_sampled_rows(cfg):
    """Full-size configs in the bench's launch configuration; the oracle recomputes sampled query rows."""
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    n, H, dh = cfg.n, cfg.H, cfg.dh
    O = pf.O.view(cfg.B, n, H, dh)
    K = pf.K.view(cfg.B, n, H, dh)
    V = pf.V.view(cfg.B, n, H, dh)
    rng = np.random.default_rng(7)
    b = cfg.B - 1
    st = np.asarray(chunk_starts(inp)[b])
    rows = sorted({0, 1, 127, 128, n - 129, n - 1} | set(rng.integers(0, n, size=26).tolist()))
    q = f64(inp["q"][b])
    ro, _ = oracle_attention_seq(q, f64(K[b]), f64(V[b]), st, n, cfg.L, cfg.mode, inp["scale"], rows)
    assert_close(cfg.dtype, f64(O[b])[rows], ro, "O (isolated, sampled)")
    rk, rv = oracle_scan_seq(inp, b)
    rk, rv = rk.reshape(n, H, dh), rv.reshape(n, H, dh)
    eo, _ = oracle_attention_seq(q, rk, rv, st, n, cfg.L, cfg.mode, inp["scale"], rows)
    extra = attn_rounding_bound(q[rows], rk, rv, eo, key_lists(n, st, cfg.L, cfg.mode, rows), inp["scale"])
    assert_close(cfg.dtype, f64(O[b])[rows], eo, "O (end to end, sampled)", extra=extra)
    assert pf.status.item() == 0


def test_value_one_gives_output_one():
    """V == 1 everywhere gives O == 1 on every row with a key (softmax weights sum to one)."""
    cfg = W.shrink(C2, B=2, n=300, D=128, H=2)
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    pf.V.fill_(1.0)
    pf.Vc.fill_(1.0)
    poison_(pf.O)
    pf.attn_step(inp["q"].cuda(), inp["scale"])
    torch.cuda.synchronize()
    pf.guard.check()
    assert_written(pf.O, "O")
    np.testing.assert_allclose(f64(pf.O), 1.0, atol=1e-2)


@pytest.mark.parametrize("cfg", [W.shrink(C2, B=2, n=520, D=128, H=2), W.shrink(W.TINY_F32_TRAIN, B=1, n=200)],
                         ids=["bf16", "f32"])
def test_attention_without_lse(cfg):
    """The LSE output is optional: without it the same O comes out, bit for bit."""
    from ssm_compressed_chunked_b200 import attamba as A
    inp = W.make_layer(cfg)
    pf = run_prefill(inp, cfg)
    H, dh = cfg.H, cfg.dh
    O2 = torch.full_like(pf.O, float("nan"))
    q = inp["q"].to(pf.O.device).reshape(-1, H, dh)
    A.chunk_attn_fwd(q, pf.K.view(-1, H, dh), pf.V.view(-1, H, dh), pf.Kc.view(-1, H, dh), pf.Vc.view(-1, H, dh),
                     pf.index, inp["scale"], O2, None, pf.status)
    torch.cuda.synchronize()
    assert pf.status.item() == 0
    assert_written(O2, "O without lse")
    assert torch.equal(O2, pf.O)
