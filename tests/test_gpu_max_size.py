"""The hot path on either side of the scan's switch to 64-bit offsets (GPU).

The scan addresses the [T, D] arrays with 32-bit element offsets while
T * D < 2^31 and with 64-bit ones beyond (a second instantiation).  Here one
sequence of n = 2^21 - 64 tokens at d_model 1024 (T * D = 2^31 - 65536, the
32-bit form) and one of n = 2^21 + 64 (T * D = 2^31 + 65536, the 64-bit form)
run through the chunk index, both scans and the attention under M_test (P =
4096, L = 64, so each query reads up to 512 chunk ends plus 64 window keys).
The oracle checks sampled chunks and query rows, the last ones among them,
where the offsets are largest.  Inputs are drawn on the device from a seeded generator
(N(0, 1), like the projected workload tensors); A and the step bias follow the
workload recipe.  Every output buffer is poisoned and guarded.
"""

import numpy as np
import pytest
import torch

from helpers import Guarded, assert_bf16_close, assert_written, f64
from oracle import attention as OA
from oracle import chunks as OC
from oracle import mask as OM
from oracle import ssm as OS
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import layer
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu

D, H, DH, NS, P, L = 1024, 16, 64, 16, 4096, 64


@pytest.mark.parametrize("n", [(1 << 21) - 64, (1 << 21) + 64], ids=["32-bit offsets", "64-bit offsets"])
def test_hot_path_at_the_offset_limit(n):
    B = 1
    T = B * n
    assert abs(T * D - 2 ** 31) == 64 * D
    bf = torch.bfloat16
    gen = torch.Generator(device="cuda").manual_seed(2024)
    rnd = lambda *shape: torch.randn(*shape, generator=gen, device="cuda", dtype=bf)  # noqa: E731
    x, dt_k, dt_v = rnd(T, D), rnd(T, D), rnd(T, D)
    q = rnd(T, H, DH)
    B_k, C_k, B_v, C_v = (rnd(T, NS) for _ in range(4))
    cpu = torch.Generator().manual_seed(2024)
    A_k, A_v = W._A(D, NS, cpu), W._A(D, NS, cpu)
    bias_k, bias_v = W._dt_bias(D, cpu), W._dt_bias(D, cpu)
    g = {k: v.cuda() for k, v in dict(A_k=A_k, A_v=A_v, bias_k=bias_k, bias_v=bias_v).items()}

    starts = OC.uniform_starts(n, P, 0)
    nch = B * A.uniform_chunk_count(n, P, 0)
    assert nch == len(starts)
    guard = Guarded()
    pf = layer.Prefill(B, n, D, H, DH, NS, nch, bf, alloc=guard)
    scale = 1.0 / DH ** 0.5
    pf.forward(x, q, dt_k, dt_v, g["bias_k"], g["bias_v"], g["A_k"], g["A_v"], B_k, C_k, B_v, C_v, None, P, 0, L,
               A.MASK_TEST, scale)
    torch.cuda.synchronize()
    assert pf.status.item() == 0
    guard.check()
    for name in ("K", "V", "Kc", "Vc", "O", "lse"):
        assert_written(getattr(pf, name), name)

    # index: the key sets of sampled queries, bit for bit, against the dense definition's row
    rows = [0, 63, 64, 4095, 4096, 4159, n // 2, n - 4097, n - 4096, n - 65, n - 2, n - 1]
    ls = pf.index.ls.cpu().numpy()
    nbb = pf.index.nbb.cpu().numpy()
    bpos = pf.index.bpos.cpu().numpy()
    key_lists = []
    for i in rows:
        ref = np.nonzero(OM.mask_row(i, n, starts, L, "test"))[0]
        got = np.concatenate([bpos[: nbb[i]], np.arange(ls[i], i + 1)])
        assert np.array_equal(got, ref), i
        key_lists.append(ref)

    # scan: sampled chunks against the oracle recurrence (the last chunks end at token T - 1)
    ends = np.append(starts[1:], n)
    for c in (0, len(starts) // 2, len(starts) - 2, len(starts) - 1):
        t0, t1 = int(starts[c]), int(ends[c])
        is_start = np.zeros(t1 - t0, dtype=bool)
        is_start[0] = True
        for s, out, outc in (("k", pf.K, pf.Kc), ("v", pf.V, pf.Vc)):
            dt = dt_k if s == "k" else dt_v
            Bm, Cm = (B_k, C_k) if s == "k" else (B_v, C_v)
            ref, _ = OS.selective_scan(f64(x[t0:t1]), f64(dt[t0:t1]), f64(g["bias_" + s]), f64(g["A_" + s]),
                                       f64(Bm[t0:t1]), f64(Cm[t0:t1]), is_start)
            assert_bf16_close(f64(out[t0:t1]), ref, f"{s} chunk {c}")
            assert torch.equal(outc[c], out[t1 - 1]), f"{s}c row {c}"

    # attention: sampled rows over the GPU's own K, V (stage-isolated), keys gathered per row
    Kv, Vv = pf.K.view(T, H, DH), pf.V.view(T, H, DH)
    O = pf.O.view(T, H, DH)
    lse = pf.lse.view(H, T).cpu().numpy()
    for i, keys in zip(rows, key_lists):
        kt = torch.from_numpy(keys).cuda()
        kr, vr = f64(Kv[kt]), f64(Vv[kt])
        qi = f64(q[i:i + 1])
        ro, rl = OA.attention_rows(qi, kr, vr, [0], [np.arange(len(keys))], scale)
        assert_bf16_close(f64(O[i:i + 1]), ro, f"O row {i}")
        assert_bf16_close(lse[:, i], rl[:, 0], f"lse row {i}")
