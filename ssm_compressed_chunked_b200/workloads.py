"""Seeded synthetic workloads for the Attamba layer hot path.

This module only draws inputs.  It holds none of the layer's arithmetic, and
none of its chunking rules: it draws the layer input and random-init weights
with the distributions below, forms the precondition projections (q = x W_Q,
dt = x W_dt, B = x W_B, C = x W_C, a plain fp32 matmul that lies outside the
hot path), rounds the results to the working dtype, and, for variable chunks,
draws the chunk lengths.  Where the chunks start, which positions end one and
what the decode cache holds are left to the caller (the tests take them from
the oracle; the library computes them itself).  Both the CUDA path and the CPU
oracle read the same rounded tensors.

Distributions (all draws from one seeded CPU ``torch.Generator`` in this order:
x, W_Q, W_dtK, W_dtV, W_BK, W_CK, W_BV, W_CV, W_O, A_K, A_V, dt_bias_K,
dt_bias_V, chunk lengths):
  x ~ N(0, 1);  projection weights ~ N(0, 1/d_model);
  A = -exp(U(log 1, log 16))  per (channel, state);
  dt_bias = delta0 + log(-expm1(-delta0)) with delta0 = exp(U(log 1e-3, log 1e-1)),
  the inverse of softplus, so that softplus(dt_bias) lies in [1e-3, 1e-1];
  variable chunk lengths ~ U{lo..hi} per sequence, drawn until their sum
  reaches n (the last one overshoots; the chunking rule cuts it at n).
There is no dataset: the pages' quality runs (WikiText-2, dclm) are not
reproduced; these tensors only have their shapes and value ranges.
"""

from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    B: int
    n: int
    D: int
    H: int
    dh: int
    N: int
    P: int               # chunk size (uniform); ignored when varlen is set
    offset: int          # cyclic chunk offset = layer_idx mod P
    L: int               # leading tokens
    mode: str            # "train" (M_train) or "test" (M_test)
    dtype: str           # "f32" or "bf16"
    seed: int
    varlen: tuple = None  # (lo, hi) chunk-length range, or None for uniform P


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    ctx: int             # context already in the cache (compressed)
    D: int
    H: int
    dh: int
    N: int
    P: int
    offset: int
    L: int
    steps: int
    seed: int
    dtype: str = "bf16"


LAYER_CONFIGS = [
    LayerConfig("tiny_f32_train", 1, 256, 128, 2, 64, 16, 4, 0, 0, "train", "f32", 0),
    LayerConfig("bf16_train_cyclic", 8, 2048, 512, 8, 64, 16, 4, 3 % 4, 4, "train", "bf16", 1),
    LayerConfig("bf16_test_P8_L64", 4, 4096, 1024, 16, 64, 16, 8, 0, 64, "test", "bf16", 2),
    LayerConfig("bf16_varlen_train", 4, 8192, 1024, 16, 64, 16, 0, 0, 32, "train", "bf16", 3, (2, 16)),
]
# the same workloads by name
TINY_F32_TRAIN, BF16_TRAIN_CYCLIC, BF16_TEST_P8_L64, BF16_VARLEN_TRAIN = LAYER_CONFIGS
DECODE_CONFIG = DecodeConfig("bf16_decode", 32, 16384, 2048, 32, 64, 16, 8, 0, 64, 128, 4)


def torch_dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def shrink(cfg, **kw):
    """Same workload recipe at other sizes (parity cases the oracle finishes in seconds)."""
    return replace(cfg, **kw)


def draw_chunk_lengths(cfg, gen):
    """Variable chunk lengths of each sequence, U{lo..hi}, drawn until their sum reaches n;
    None for uniform chunks (nothing is drawn)."""
    if cfg.varlen is None:
        return None
    lo, hi = cfg.varlen
    out = []
    for _ in range(cfg.B):
        lengths, total = [], 0
        while total < cfg.n:
            ln = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
            lengths.append(ln)
            total += ln
        out.append(lengths)
    return out


def _dt_bias(D, gen):
    lo, hi = math.log(1e-3), math.log(1e-1)
    d0 = torch.exp(torch.rand(D, generator=gen, dtype=torch.float64) * (hi - lo) + lo)
    return (d0 + torch.log(-torch.expm1(-d0))).float()


def _A(D, N, gen):
    return -torch.exp(torch.rand(D, N, generator=gen) * math.log(16.0))


def draw_weights(D, H, dh, N, gen):
    s = 1.0 / math.sqrt(D)
    W = {}
    for name, cols in (("Q", H * dh), ("dtK", D), ("dtV", D), ("BK", N), ("CK", N),
                       ("BV", N), ("CV", N), ("O", D)):
        W[name] = torch.randn(D, cols, generator=gen) * s
    return W


def make_layer(cfg):
    """All hot-path inputs of one prefill config, rounded to cfg.dtype, on the CPU.

    Returns a dict with  x, dt_k, dt_v [B, n, D];  q [B, n, H, dh];
    B_k, C_k, B_v, C_v [B, n, N];  A_k, A_v [D, N] f32;  bias_k, bias_v [D] f32;
    lengths (variable chunks: the drawn chunk lengths per sequence; else None);
    scale = 1/sqrt(dh).
    """
    gen = torch.Generator().manual_seed(cfg.seed)
    Bsz, n, D, H, dh, N = cfg.B, cfg.n, cfg.D, cfg.H, cfg.dh, cfg.N
    x = torch.randn(Bsz, n, D, generator=gen)
    W = draw_weights(D, H, dh, N, gen)
    A_k, A_v = _A(D, N, gen), _A(D, N, gen)
    bias_k, bias_v = _dt_bias(D, gen), _dt_bias(D, gen)
    lengths = draw_chunk_lengths(cfg, gen)
    dt = torch_dtype(cfg.dtype)
    xf = x.reshape(Bsz * n, D)
    proj = {k: (xf @ W[k]) for k in ("Q", "dtK", "dtV", "BK", "CK", "BV", "CV")}
    r = lambda t, *shape: t.reshape(*shape).to(dt).contiguous()
    return dict(
        cfg=cfg,
        x=r(x, Bsz, n, D),
        q=r(proj["Q"], Bsz, n, H, dh),
        dt_k=r(proj["dtK"], Bsz, n, D), dt_v=r(proj["dtV"], Bsz, n, D),
        B_k=r(proj["BK"], Bsz, n, N), C_k=r(proj["CK"], Bsz, n, N),
        B_v=r(proj["BV"], Bsz, n, N), C_v=r(proj["CV"], Bsz, n, N),
        A_k=A_k.contiguous(), A_v=A_v.contiguous(),
        bias_k=bias_k.contiguous(), bias_v=bias_v.contiguous(),
        lengths=lengths,
        scale=1.0 / math.sqrt(dh),
    )


def decode_capacity(cfg):
    """Boundary slots per sequence: every chunk end the context and the decoded steps can hold."""
    return (cfg.ctx + cfg.steps) // cfg.P + 2


def make_decode(cfg):
    """Random contents for a decode cache of ``cfg.ctx`` compressed tokens plus ``cfg.steps``
    step inputs (CPU).

    Drawn here: candidate boundary keys/values for every one of the cache's boundary slots,
    keys/values for the L ring slots, and the SSM states, all ~ N(0, 1); step inputs
    x_t ~ N(0, 1) projected like the prefill.  Which slots hold a boundary (the positions
    below ctx that end a chunk) and which ring slots repeat a boundary is the chunking rule,
    left to the caller.

    Returns Kb, Vb [B, H, cap, dh];  Kr, Vr [B, H, L, dh];  state [2, B, N, D] f32;
    x, dt_k, dt_v [steps, B, D];  q [steps, B, H, dh];  B_k .. C_v [steps, B, N];
    A_k, A_v, bias_k, bias_v as in make_layer;  cap;  scale.
    """
    gen = torch.Generator().manual_seed(cfg.seed)
    Bsz, D, H, dh, N, L = cfg.B, cfg.D, cfg.H, cfg.dh, cfg.N, cfg.L
    dt = torch_dtype(cfg.dtype)
    xs = torch.randn(cfg.steps, Bsz, D, generator=gen)
    W = draw_weights(D, H, dh, N, gen)
    A_k, A_v = _A(D, N, gen), _A(D, N, gen)
    bias_k, bias_v = _dt_bias(D, gen), _dt_bias(D, gen)
    cap = decode_capacity(cfg)
    Kb = torch.randn(Bsz, H, cap, dh, generator=gen).to(dt)
    Vb = torch.randn(Bsz, H, cap, dh, generator=gen).to(dt)
    Kr = torch.randn(Bsz, H, L, dh, generator=gen).to(dt)
    Vr = torch.randn(Bsz, H, L, dh, generator=gen).to(dt)
    state = torch.randn(2, Bsz, N, D, generator=gen)
    xf = xs.reshape(cfg.steps * Bsz, D)
    proj = {k: (xf @ W[k]) for k in ("Q", "dtK", "dtV", "BK", "CK", "BV", "CV")}
    r = lambda t, *shape: t.reshape(*shape).to(dt).contiguous()
    S = cfg.steps
    return dict(
        cfg=cfg, cap=cap,
        state=state.contiguous(),                # [2, B, N, D] f32 (state-major per channel)
        Kb=Kb, Vb=Vb, Kr=Kr, Vr=Vr,
        x=r(xs, S, Bsz, D),
        q=r(proj["Q"], S, Bsz, H, dh),
        dt_k=r(proj["dtK"], S, Bsz, D), dt_v=r(proj["dtV"], S, Bsz, D),
        B_k=r(proj["BK"], S, Bsz, N), C_k=r(proj["CK"], S, Bsz, N),
        B_v=r(proj["BV"], S, Bsz, N), C_v=r(proj["CV"], S, Bsz, N),
        A_k=A_k.contiguous(), A_v=A_v.contiguous(),
        bias_k=bias_k.contiguous(), bias_v=bias_v.contiguous(),
        scale=1.0 / math.sqrt(dh),
    )
