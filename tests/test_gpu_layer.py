"""The whole layer with its projections (layer.Layer) against the oracle, stage by stage (GPU).

x -> one GEMM for the seven input projections -> chunk index -> the two scans -> attention ->
y = O W_O.  Each stage is compared with the oracle fed that stage's inputs as the GPU produced
them (bf16), so the tolerances are the single-stage ones and a projection segment wired to the
wrong consumer fails its check: every projection against x W^T of its own weight block, K and V
against the oracle scan of x with the GPU's dt, B, C, O against the oracle attention of the GPU's
q, K, V under the mask of the layer's chunking, and y against O W_O.  Every output buffer is
poisoned and guarded, and is checked to be written in full.
"""

import math

import numpy as np
import pytest
import torch

from helpers import BF16_ATOL, Guarded, assert_bf16_close, assert_written, f64, oracle_attention_seq
from oracle import chunks as OC
from oracle import projection as OP
from oracle import ssm as OS
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import layer
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu

DH = 64


def _gemm_check(Y, ref, X, Wm, what):
    """bf16 rounding of the result (half an ulp, 2^-9 relative) plus the fp32 accumulation
    error bound of a K-term dot product, sum |x||w| K 2^-24."""
    mag = np.abs(f64(X)) @ np.abs(f64(Wm)).T
    bound = 2.0 ** -8 * np.abs(ref) + X.shape[1] * 2.0 ** -24 * mag + 1e-6
    err = np.abs(f64(Y) - ref)
    k = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"{what}: err {err[k]:.3e} > bound {bound[k]:.3e} at {k}"


# (B, n, H, N, chunking, L, mask): D = H * 64.  n = 300 leaves a partial 128-query tile; the
# variable chunking passes chunk offsets to the layer instead of (P, offset)
CASES = [
    (1, 512, 16, 16, ("uniform", 8, 0), 64, "test"),   # the bench workload's width and mask, 512 tokens
    (2, 300, 2, 16, ("uniform", 8, 3), 16, "test"),
    (1, 257, 4, 32, ("uniform", 4, 0), 4, "train"),
    (2, 200, 2, 16, ("varlen", 2, 12), 8, "train"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_n{c[1]}_H{c[2]}_N{c[3]}_{c[4][0]}_{c[6]}")
def test_layer_stages_match_oracle(case):
    B, n, H, N, chunking, L, mode = case
    D = H * DH
    T = B * n
    bf = torch.bfloat16
    gen = torch.Generator().manual_seed(1000 + n)
    s = 1.0 / math.sqrt(D)
    shapes = {"W_Q": (H * DH, D), "W_dtK": (D, D), "W_dtV": (D, D), "W_BK": (N, D), "W_CK": (N, D),
              "W_BV": (N, D), "W_CV": (N, D), "W_O": (D, H * DH)}
    w = {k: (torch.randn(*shp, generator=gen) * s).to(bf) for k, shp in shapes.items()}
    w["bias_k"], w["bias_v"] = W._dt_bias(D, gen), W._dt_bias(D, gen)
    w["A_k"], w["A_v"] = W._A(D, N, gen), W._A(D, N, gen)
    x = torch.randn(T, D, generator=gen).to(bf)
    scale = 1.0 / math.sqrt(DH)

    if chunking[0] == "uniform":
        _, P, offset = chunking
        starts = [OC.uniform_starts(n, P, offset) for _ in range(B)]
        cu_in, n_chunks = None, None
    else:
        _, lo, hi = chunking
        P, offset = 1, 0
        starts = []
        for _ in range(B):
            lengths, total = [], 0
            while total < n:
                ln = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
                lengths.append(ln)
                total += ln
            starts.append(OC.varlen_starts(lengths, n))
        cu = OC.flatten_batch(starts, n).astype(np.int32)
        cu_in, n_chunks = torch.from_numpy(cu).cuda(), len(cu) - 1

    guard = Guarded()
    mcode = A.MASK_TEST if mode == "test" else A.MASK_TRAIN
    lay = layer.Layer(B, n, D, H, DH, N, {k: v.cuda() for k, v in w.items()}, P, offset, L, mcode, scale,
                      n_chunks=n_chunks, alloc=guard)
    y = lay.forward(x.cuda(), cu_in)
    torch.cuda.synchronize()
    assert lay.status.item() == 0
    guard.check()
    pf = lay.prefill
    pr = lay.projections
    for name, t in list(pr.items()) + [("K", pf.K), ("V", pf.V), ("Kc", pf.Kc), ("Vc", pf.Vc), ("O", pf.O),
                                       ("lse", pf.lse), ("y", y)]:
        assert_written(t, name)

    # 1. the seven input projections, each against its own weight block
    for name in layer.INPUT_PROJECTIONS:
        _gemm_check(pr[name[2:]].cpu(), OP.project(f64(x), f64(w[name])), x, w[name], name)

    # 2. the scans, from x and the GPU's dt, B, C
    for b in range(B):
        rows = slice(b * n, (b + 1) * n)
        is_start = OC.is_start_mask(starts[b], n)
        for ssm, out in (("K", pf.K), ("V", pf.V)):
            sfx = ssm.lower()
            ref, _ = OS.selective_scan(f64(x[rows]), f64(pr["dt" + ssm][rows]), f64(w["bias_" + sfx]),
                                       f64(w["A_" + sfx]), f64(pr["B" + ssm][rows]), f64(pr["C" + ssm][rows]),
                                       is_start)
            assert_bf16_close(f64(out[rows]), ref, f"{ssm} of sequence {b}")

    # 3. the attention, from the GPU's q, K, V
    for b in range(B):
        rows = slice(b * n, (b + 1) * n)
        q = f64(pr["Q"][rows]).reshape(n, H, DH)
        K = f64(pf.K[rows]).reshape(n, H, DH)
        V = f64(pf.V[rows]).reshape(n, H, DH)
        ro, _ = oracle_attention_seq(q, K, V, np.asarray(starts[b]), n, L, mode, scale)
        assert_bf16_close(f64(pf.O.view(T, H, DH)[rows]), ro, f"O of sequence {b}")

    # 4. the output projection, from the GPU's O
    Ot = pf.O.view(T, H * DH).cpu()
    _gemm_check(y.cpu(), OP.project(f64(Ot), f64(w["W_O"])), Ot, w["W_O"], "y")


@pytest.mark.parametrize("n0", [0, 120], ids=["from_empty_cache", "after_prefill_handoff"])
def test_layer_decode_continues_its_prefill(n0):
    """Decoding through the layer (Layer.decode_step) from an empty cache, or from the cache a
    Layer.forward over the first n0 tokens leaves (Layer.cache_from_prefill): at every position t the
    step's attention output is the M_test prefill row t of a Layer.forward over the whole sequence
    (itself checked against the oracle above) within bf16 rounding, and the step's seven projections
    and y_t match the oracle's products of the step's own inputs."""
    B, steps, H, N, P, offset, L = 2, 40, 2, 16, 8, 3, 16
    n = n0 + steps
    D = H * DH
    bf = torch.bfloat16
    gen = torch.Generator().manual_seed(77 + n0)
    s = 1.0 / math.sqrt(D)
    shapes = {"W_Q": (H * DH, D), "W_dtK": (D, D), "W_dtV": (D, D), "W_BK": (N, D), "W_CK": (N, D),
              "W_BV": (N, D), "W_CV": (N, D), "W_O": (D, H * DH)}
    w = {k: (torch.randn(*shp, generator=gen) * s).to(bf) for k, shp in shapes.items()}
    w["bias_k"], w["bias_v"] = W._dt_bias(D, gen), W._dt_bias(D, gen)
    w["A_k"], w["A_v"] = W._A(D, N, gen), W._A(D, N, gen)
    wg = {k: v.cuda() for k, v in w.items()}
    x = torch.randn(B, n, D, generator=gen).to(bf)
    scale = 1.0 / math.sqrt(DH)
    args = (H, DH, N, wg, P, offset, L, A.MASK_TEST, scale)

    full = layer.Layer(B, n, D, *args)
    full.forward(x.view(B * n, D).cuda())
    O_full = full.prefill.O.view(B, n, H, DH)
    cap = n // P + 2
    if n0 == 0:
        dec = full
        cache = dec.new_cache(cap)
    else:
        dec = layer.Layer(B, n0, D, *args)
        xp = x[:, :n0].reshape(B * n0, D).contiguous().cuda()
        dec.forward(xp)
        cache = dec.new_cache(cap)
        dec.cache_from_prefill(cache, xp)
    for t in range(n0, n):
        xt = x[:, t].contiguous()
        y_t = dec.decode_step(cache, xt.cuda())
        torch.cuda.synchronize()
        err = (dec.o_t.float() - O_full[:, t].float()).abs().max().item()
        assert err <= BF16_ATOL, f"o_t at position {t}: {err} from the prefill row"
        sp = dec.step_projections
        for name in layer.INPUT_PROJECTIONS:
            _gemm_check(sp[name[2:]].cpu(), OP.project(f64(xt), f64(w[name])), xt, w[name], f"{name} at {t}")
        ot = dec.o_t.view(B, H * DH).cpu()
        _gemm_check(y_t.cpu(), OP.project(f64(ot), f64(w["W_O"])), ot, w["W_O"], f"y_t at {t}")
    assert full.status.item() == 0 and dec.status.item() == 0
    assert (cache.pos.cpu() == n).all()
