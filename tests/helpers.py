"""Shared test plumbing: run the CUDA path on a workload and run the oracle on the same inputs."""

import numpy as np
import torch

from oracle import attention as OA
from oracle import chunks as OC
from oracle import mask as OM
from oracle import ssm as OS
from ssm_compressed_chunked_b200 import layer
from ssm_compressed_chunked_b200 import workloads as W

BF16_ATOL = 2e-2       # bf16 outputs, fp32 accumulation (stated tolerance)
BF16_HALF_ULP = 2.0 ** -8   # a bf16 value is within 2^-8 |x| of x (8-bit significand, round to nearest)
F32_RTOL = 1e-4        # fp32 outputs: |gpu - ref| <= 1e-4 * (|ref| + rms(ref))

# Reading of the stated bf16 tolerance: 2e-2 absolute bounds the arithmetic
# error (fp32 accumulation) on top of the rounding that storing a value in bf16
# cannot avoid.  A stored bf16 output is compared with
#     |gpu - ref| <= 2e-2 + 2^-8 |ref|,
# and an output computed from stored bf16 intermediates (the attention over the
# bf16 K and V the scan wrote) adds the first-order effect of that rounding,
# computed from the oracle's own values (see attn_rounding_bound).


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_f32_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = F32_RTOL * (np.abs(ref) + rms)
    worst = np.max(err - bound) if err.size else -1
    assert worst <= 0, f"{what}: max excess {worst:.3e}, max err {err.max():.3e}, rms(ref) {rms:.3e}"


def assert_bf16_close(got, ref, what="", extra=0.0, rel=BF16_HALF_ULP):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = BF16_ATOL + rel * np.abs(ref) + extra
    k = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (f"{what}: err {err[k]:.3e} > bound {bound[k]:.3e} at {k} "
                                  f"(ref {ref[k]:.4f}, got {got[k]:.4f}); max abs err {err.max():.3e}")


def assert_close(dtype, got, ref, what="", extra=0.0):
    if dtype == "f32":
        assert_f32_close(got, ref, what)
    else:
        assert_bf16_close(got, ref, what, extra=extra)


def attn_rounding_bound(q, K, V, O, key_lists, scale):
    """First-order effect on O of storing K and V in bf16 (each entry moved by <= 2^-8 of itself).

    For query i, head h and key set S:  O = sum_j p_j v_j with p = softmax(s),
    s_j = scale q.k_j.  A change dv_j moves O by <= max_j |dv_j|; a change dk_j
    moves s_j by ds_j <= scale sum_d |q_d| |dk_jd| and O by <= max_j |v_j - O| max_j |ds_j|.
    Returns the bound per (row, head, dim) as an array shaped like O.
    """
    out = np.zeros_like(O)
    for r, keys in enumerate(key_lists):
        keys = np.asarray(keys, dtype=np.int64)
        if keys.size == 0:
            continue
        k = K[keys]                       # [|S|, H, dh]
        v = V[keys]
        ds = scale * BF16_HALF_ULP * np.einsum("hd,jhd->jh", np.abs(q[r]), np.abs(k))   # [|S|, H]
        dv = BF16_HALF_ULP * np.abs(v).max(axis=0)                                      # [H, dh]
        spread = np.abs(v - O[r][None]).max(axis=0)                                     # [H, dh]
        out[r] = dv + spread * ds.max(axis=0)[:, None]
    return out


def to_gpu(inp):
    out = {}
    for k, v in inp.items():
        out[k] = v.cuda() if isinstance(v, torch.Tensor) else v
    out["cu_t"] = torch.from_numpy(inp["cu"]).cuda()
    return out


def run_prefill(inp, cfg):
    """CUDA path on a workload dict (CPU tensors); returns the Prefill object (device buffers)."""
    g = to_gpu(inp)
    nch = layer.n_chunks_of(cfg, inp["cu"])
    pf = layer.Prefill(cfg.B, cfg.n, cfg.D, cfg.H, cfg.dh, cfg.N, nch, W.torch_dtype(cfg.dtype))
    cu_in = g["cu_t"] if cfg.varlen is not None else None
    P = cfg.P if cfg.varlen is None else 1
    pf.forward(g["x"], g["q"], g["dt_k"], g["dt_v"], g["bias_k"], g["bias_v"], g["A_k"], g["A_v"],
               g["B_k"], g["C_k"], g["B_v"], g["C_v"], cu_in, P, cfg.offset, cfg.L, layer.mode_code(cfg.mode),
               inp["scale"])
    torch.cuda.synchronize()
    return pf


def oracle_scan_seq(inp, b, t0=None, t1=None):
    """Oracle K, V [len, D] of sequence b over positions [t0, t1) (t0 must start a chunk)."""
    cfg = inp["cfg"]
    n = cfg.n
    t0 = 0 if t0 is None else t0
    t1 = n if t1 is None else t1
    starts = np.asarray(inp["starts"][b])
    is_start = OC.is_start_mask(starts, n)[t0:t1]
    assert is_start[0]
    sl = slice(t0, t1)
    out = []
    for s in ("k", "v"):
        y, _ = OS.selective_scan(f64(inp["x"][b, sl]), f64(inp["dt_" + s][b, sl]), f64(inp["bias_" + s]),
                                 f64(inp["A_" + s]), f64(inp["B_" + s][b, sl]), f64(inp["C_" + s][b, sl]),
                                 is_start)
        out.append(y)
    return out


def key_lists(n, starts, L, mode, rows):
    return [np.nonzero(OM.mask_row(i, n, starts, L, mode))[0] for i in rows]


def oracle_attention_seq(q, K, V, starts, n, L, mode, scale, rows=None):
    """Oracle attention of one sequence (q, K, V as [n, H, dh] float64); rows=None means all."""
    if rows is None:
        return OA.masked_attention(q, K, V, OM.dense_mask(n, starts, L, mode), scale)
    return OA.attention_rows(q, K, V, rows, key_lists(n, starts, L, mode, rows), scale)
