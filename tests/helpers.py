"""Shared test plumbing: run the CUDA path on a workload and run the oracle on the same inputs.

The chunk layout of a workload (where its chunks start, which positions end
one, what a decode cache holds) always comes from the oracle's own rules
(``oracle.chunks``, ``oracle.decode``); the workload generator only draws
random values and chunk lengths.

Every buffer a kernel writes in these tests is poisoned first and placed between
two guard regions (``Guarded``): outputs start as a NaN canary (0xA5A5A5A5 for
int32), so a value a kernel leaves unwritten fails the comparison instead of
passing on memory an earlier test left behind, and a write before the start or
past the end of an array shows up as a changed guard.  These stand in for a
memory checker.
"""

import math

import numpy as np
import torch

from oracle import attention as OA
from oracle import chunks as OC
from oracle import decode as OD
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


# ------------------------------------------------------------------ chunk layout from the oracle
def chunk_starts(inp):
    """Sequence-relative chunk starts of each sequence of a workload, by the oracle's rules:
    uniform chunks (size P, cyclic offset) or the drawn variable lengths cut at n."""
    cfg = inp["cfg"]
    if cfg.varlen is None:
        return [OC.uniform_starts(cfg.n, cfg.P, cfg.offset) for _ in range(cfg.B)]
    return [OC.varlen_starts(lengths, cfg.n) for lengths in inp["lengths"]]


def cu_of(inp):
    """cu_seqlens-style chunk starts over the B sequences laid end to end (int32)."""
    return OC.flatten_batch(chunk_starts(inp), inp["cfg"].n).astype(np.int32)


# ------------------------------------------------------------------ poisoned, guarded outputs
GUARD = 256   # guard elements after every array
_CANARY = {torch.bfloat16: (torch.int16, 0x7FA5),            # a NaN
           torch.float32: (torch.int32, 0x7FA5A5A5),          # a NaN
           torch.int32: (torch.int32, -0x5A5A5A5B)}           # 0xA5A5A5A5, never a valid index


def poison_(t):
    """Fill t with its dtype's canary (NaN for floats, 0xA5A5A5A5 for int32) in place."""
    iv, pat = _CANARY[t.dtype]
    t.view(iv).fill_(pat)
    return t


class Guarded:
    """Allocator of poisoned output buffers, each between two runs of GUARD canary elements.

    The array starts GUARD elements into its buffer (512 bytes or more, so every 16-byte alignment the
    library asks for holds)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.bufs = []

    def __call__(self, shape, dtype):
        numel = math.prod(shape)
        buf = poison_(torch.empty(numel + 2 * GUARD, dtype=dtype, device=self.device))
        self.bufs.append((buf, numel))
        return buf[GUARD:GUARD + numel].view(shape)

    def check(self):
        """Both guard regions of every array still hold the canary (no write before its start or past
        its end)."""
        for buf, numel in self.bufs:
            iv, pat = _CANARY[buf.dtype]
            for where, g in (("before", buf[:GUARD]), ("after", buf[GUARD + numel:])):
                assert bool((g.view(iv) == pat).all()), \
                    f"guard {where} a {numel}-element {buf.dtype} array was written"


def assert_written(t, what):
    """No element of t still holds the canary: the kernel wrote all of it."""
    if t.dtype == torch.int32:
        assert bool((t != _CANARY[torch.int32][1]).all()), f"{what}: entries left unwritten"
    else:
        assert not bool(torch.isnan(t).any()), f"{what}: NaN (unwritten) entries"


def to_gpu(inp):
    out = {}
    for k, v in inp.items():
        out[k] = v.cuda() if isinstance(v, torch.Tensor) else v
    out["cu"] = cu_of(inp)
    out["cu_t"] = torch.from_numpy(out["cu"]).cuda()
    return out


def run_prefill(inp, cfg):
    """CUDA path on a workload dict (CPU tensors) into poisoned, guarded buffers; checks the guards
    and that every output element was written, and returns the Prefill object (device buffers)."""
    g = to_gpu(inp)
    nch = layer.n_chunks_of(cfg, g["cu"])
    guard = Guarded()
    pf = layer.Prefill(cfg.B, cfg.n, cfg.D, cfg.H, cfg.dh, cfg.N, nch, W.torch_dtype(cfg.dtype), alloc=guard)
    cu_in = g["cu_t"] if cfg.varlen is not None else None
    P = cfg.P if cfg.varlen is None else 1
    pf.forward(g["x"], g["q"], g["dt_k"], g["dt_v"], g["bias_k"], g["bias_v"], g["A_k"], g["A_v"],
               g["B_k"], g["C_k"], g["B_v"], g["C_v"], cu_in, P, cfg.offset, cfg.L, layer.mode_code(cfg.mode),
               inp["scale"])
    torch.cuda.synchronize()
    pf.guard = guard
    guard.check()
    for name in ("K", "V", "Kc", "Vc", "O", "lse"):
        assert_written(getattr(pf, name), name)
    for name in ("cu", "bpos", "bptr", "ls", "nbb"):
        assert_written(getattr(pf.index, name), "index." + name)
    return pf


def oracle_scan_seq(inp, b, t0=None, t1=None):
    """Oracle K, V [len, D] of sequence b over positions [t0, t1) (t0 must start a chunk)."""
    cfg = inp["cfg"]
    n = cfg.n
    t0 = 0 if t0 is None else t0
    t1 = n if t1 is None else t1
    starts = np.asarray(chunk_starts(inp)[b])
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


# ------------------------------------------------------------------ decode caches
def decode_cache_contents(dec):
    """The synthetic decode cache of ``W.make_decode`` laid out by the oracle's chunk-end rule:
    boundaries at the positions below ctx that end a chunk (their rows from the drawn candidates,
    the rows past them poisoned with NaN so a read past nb shows), ring slots of window positions
    that are boundaries holding the boundary's key/value, pos = ctx.  CPU tensors."""
    cfg = dec["cfg"]
    bpos = [p for p in range(cfg.ctx) if OD.is_chunk_end(p, cfg.P, cfg.offset)]
    nb, cap = len(bpos), dec["cap"]
    assert nb <= cap
    Kb, Vb = dec["Kb"].clone(), dec["Vb"].clone()
    Kb[:, :, nb:] = float("nan")
    Vb[:, :, nb:] = float("nan")
    Kr, Vr = dec["Kr"].clone(), dec["Vr"].clone()
    for k, p in enumerate(bpos):
        if p >= cfg.ctx - cfg.L:
            Kr[:, :, p % cfg.L] = Kb[:, :, k]
            Vr[:, :, p % cfg.L] = Vb[:, :, k]
    bp = torch.full((cfg.B, cap), -1, dtype=torch.int32)
    bp[:, :nb] = torch.tensor(bpos, dtype=torch.int32)
    return dict(state=dec["state"].clone(), Kb=Kb, Vb=Vb, bpos=bp, Kr=Kr, Vr=Vr,
                nb=torch.full((cfg.B,), nb, dtype=torch.int32),
                pos=torch.full((cfg.B,), cfg.ctx, dtype=torch.int32))


_CACHE_ARRAYS = ("state", "Kb", "Vb", "bpos", "Kr", "Vr", "nb", "pos")


def gpu_cache(contents, P, offset, guard=None):
    """A device cache (attamba.Cache) holding copies of ``contents``; each array inside a guarded
    buffer when ``guard`` (a Guarded) is given."""
    from ssm_compressed_chunked_b200 import attamba as A
    arrs = {}
    for k in _CACHE_ARRAYS:
        src = contents[k]
        if guard is None:
            arrs[k] = src.cuda().clone()
        else:
            t = guard(tuple(src.shape), src.dtype)
            t.copy_(src)
            arrs[k] = t
    return A.Cache(*(arrs[k] for k in _CACHE_ARRAYS), P, offset)


def empty_cache_contents(B, H, dh, N, L, cap):
    """An empty decode cache (no boundaries, position 0); unwritten rows poisoned with NaN / -1."""
    D = H * dh
    bf = torch.bfloat16
    return dict(state=torch.full((2, B, N, D), float("nan")),
                Kb=torch.full((B, H, cap, dh), float("nan"), dtype=bf),
                Vb=torch.full((B, H, cap, dh), float("nan"), dtype=bf),
                bpos=torch.full((B, cap), -1, dtype=torch.int32),
                Kr=torch.full((B, H, L, dh), float("nan"), dtype=bf),
                Vr=torch.full((B, H, L, dh), float("nan"), dtype=bf),
                nb=torch.zeros(B, dtype=torch.int32), pos=torch.zeros(B, dtype=torch.int32))


def oracle_cache(contents, cfg, rows):
    """A cache's contents (CPU tensors) in the oracle's format, for the batch rows ``rows``."""
    c = OD.DecodeCache(len(rows), cfg.H, cfg.dh, cfg.N, cfg.P, cfg.offset, cfg.L)
    c.state = np.transpose(f64(contents["state"][:, rows]), (0, 1, 3, 2)).copy()
    for r, b in enumerate(rows):
        nb = int(contents["nb"][b])
        t = int(contents["pos"][b])
        c.bpos[r] = contents["bpos"][b, :nb].tolist()
        Kb = f64(contents["Kb"][b, :, :nb])
        Vb = f64(contents["Vb"][b, :, :nb])
        c.Kb[r] = [Kb[:, k] for k in range(nb)]
        c.Vb[r] = [Vb[:, k] for k in range(nb)]
        for p in range(max(0, t - cfg.L), t):
            c.ring[r][p] = (f64(contents["Kr"][b, :, p % cfg.L]), f64(contents["Vr"][b, :, p % cfg.L]))
        c.pos[r] = t
    return c


def oracle_step(oc, dec_or_inp, s, rows, scale, col=None):
    """One oracle decode step for the batch rows ``rows`` on step s's inputs.

    ``dec_or_inp`` holds per-step arrays [steps, B, ...] (col None) or prefill arrays
    [B, n, ...] read at position ``col``."""
    def sel(name):
        t = dec_or_inp[name]
        return f64(t[s][rows]) if col is None else f64(t[rows, col])
    return oc.step(sel("q"), sel("x"), np.stack([sel("dt_k"), sel("dt_v")]),
                   np.stack([f64(dec_or_inp["bias_k"]), f64(dec_or_inp["bias_v"])]),
                   np.stack([f64(dec_or_inp["A_k"]), f64(dec_or_inp["A_v"])]),
                   np.stack([sel("B_k"), sel("B_v")]), np.stack([sel("C_k"), sel("C_v")]), scale)


def decode_rounding_bound(oc, r, q, o_ref, ctx, scale):
    """First-order effect on a decode output of keys the GPU stored in bf16 while the oracle keeps
    them in float64: the keys and values at positions >= ctx (those the GPU computed; rows of a
    synthetic bf16 cache are the same on both sides).  Same rule as the prefill attention's: a
    change dv moves o by at most max |dv|, a change dk moves a score by at most scale sum |q| |dk|
    and o by at most max |v - o| times that.  Returns [H, dh] for batch row r of the oracle cache."""
    t = oc.pos[r] - 1
    lo = max(0, t - oc.L + 1)
    ks, vs = [], []
    for p, kk, vv in zip(oc.bpos[r], oc.Kb[r], oc.Vb[r]):
        if ctx <= p < lo:
            ks.append(kk)
            vs.append(vv)
    for p in range(max(lo, ctx), t + 1):
        kk, vv = oc.ring[r][p]
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
