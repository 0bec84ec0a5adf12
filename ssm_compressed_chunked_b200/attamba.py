"""ctypes binding of libattamba.so (argument marshalling only).

Every function here has the name of the C entry point it calls (without the
``attamba_`` prefix), checks that the torch tensors it is handed are CUDA,
contiguous and of the right dtype, passes their device pointers and the
current CUDA stream, and raises ``AttambaError`` on a non-OK status.  All
arithmetic happens in the library's kernels; there is no fallback path: if the
library is missing or a tensor is on the CPU, the call raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# ATTAMBA_LIBRARY=checked selects the bounds-checked build (libattamba_checked.so): the same kernels
# with every index tested against its array, a failure reported as DEV_BOUNDS in the status word
LIB_PATH = os.path.join(_HERE, "libattamba_checked.so" if os.environ.get("ATTAMBA_LIBRARY") == "checked"
                        else "libattamba.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA = 0, 1, 2, 3
F32, BF16 = 0, 1
MASK_TRAIN, MASK_TEST = 0, 1
DEV_BAD_CHUNKS, DEV_CACHE_FULL, DEV_TIMEOUT, DEV_BOUNDS = 0x1, 0x2, 0x4, 0x8

# every symbol include/attamba.h declares
EXPORTS = ("attamba_version", "attamba_status_string", "attamba_last_error",
           "attamba_uniform_chunk_count", "attamba_chunk_index", "attamba_kv_ssm_scan",
           "attamba_chunk_attn_fwd", "attamba_cache_bytes", "attamba_selftest_wait_timeout", "attamba_decode_workspace_size", "attamba_decode_step",
           "attamba_decode_step_noalloc", "attamba_cache_from_prefill",
           "attamba_kv_ssm_scan_u", "attamba_proj_gemm")


class AttambaError(RuntimeError):
    pass


class IndexT(ctypes.Structure):
    _fields_ = [("cu", ctypes.c_void_p), ("bpos", ctypes.c_void_p), ("bptr", ctypes.c_void_p),
                ("ls", ctypes.c_void_p), ("nbb", ctypes.c_void_p),
                ("n_chunks", ctypes.c_int32), ("B", ctypes.c_int32), ("n", ctypes.c_int32)]


class ProjSegT(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("col0", ctypes.c_int32), ("width", ctypes.c_int32)]


class CacheT(ctypes.Structure):
    _fields_ = [("state", ctypes.c_void_p), ("Kb", ctypes.c_void_p), ("Vb", ctypes.c_void_p),
                ("bpos", ctypes.c_void_p), ("Kr", ctypes.c_void_p), ("Vr", ctypes.c_void_p),
                ("nb", ctypes.c_void_p), ("pos", ctypes.c_void_p)] + \
               [(k, ctypes.c_int32) for k in ("B", "H", "dh", "N", "P", "offset", "L", "cap")]


_lib = None


def load():
    """Load the library once (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise AttambaError(f"{LIB_PATH} is missing: build it with python -m ssm_compressed_chunked_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    L.attamba_version.restype = ctypes.c_char_p
    L.attamba_status_string.restype = ctypes.c_char_p
    L.attamba_status_string.argtypes = [ctypes.c_int]
    L.attamba_last_error.restype = ctypes.c_char_p
    L.attamba_uniform_chunk_count.restype = i32
    L.attamba_uniform_chunk_count.argtypes = [i32, i32, i32]
    L.attamba_chunk_index.restype = ctypes.c_int
    L.attamba_chunk_index.argtypes = [vp, i32, i32, i32, i32, i32, i32, ctypes.c_int,
                                      ctypes.POINTER(IndexT), vp, vp]
    L.attamba_kv_ssm_scan.restype = ctypes.c_int
    L.attamba_kv_ssm_scan.argtypes = [ctypes.c_int] + [vp] * 12 + [i32, i64, i32, i32] + [vp] * 4 + [vp, vp]
    L.attamba_proj_gemm.restype = ctypes.c_int
    L.attamba_proj_gemm.argtypes = [ctypes.c_int, vp, vp, i64, i32, i32, ctypes.POINTER(ProjSegT), i32, vp, vp]
    L.attamba_kv_ssm_scan_u.restype = ctypes.c_int
    L.attamba_kv_ssm_scan_u.argtypes = [ctypes.c_int] + [vp] * 13 + [i32, i64, i32, i32] + [vp] * 4 + [vp, vp]
    L.attamba_chunk_attn_fwd.restype = ctypes.c_int
    L.attamba_chunk_attn_fwd.argtypes = [ctypes.c_int, vp, vp, vp, vp, vp, ctypes.POINTER(IndexT),
                                         i32, i32, f32, vp, vp, vp, vp]
    L.attamba_selftest_wait_timeout.restype = ctypes.c_int
    L.attamba_selftest_wait_timeout.argtypes = [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    L.attamba_cache_bytes.restype = sz
    L.attamba_cache_bytes.argtypes = [ctypes.POINTER(CacheT)]
    L.attamba_decode_workspace_size.restype = sz
    L.attamba_decode_workspace_size.argtypes = [ctypes.POINTER(CacheT)]
    L.attamba_decode_step.restype = ctypes.c_int
    L.attamba_decode_step.argtypes = [ctypes.c_int, ctypes.POINTER(CacheT)] + [vp] * 12 + \
                                     [f32, vp, vp, sz, vp, vp]
    L.attamba_decode_step_noalloc.restype = ctypes.c_int
    L.attamba_decode_step_noalloc.argtypes = [ctypes.c_int, ctypes.POINTER(CacheT)] + [vp] * 12 + [f32, vp, vp, vp]
    L.attamba_cache_from_prefill.restype = ctypes.c_int
    L.attamba_cache_from_prefill.argtypes = [ctypes.c_int, ctypes.POINTER(CacheT)] + [vp] * 13 + [i32, vp, vp]
    _lib = L
    return L


def _check(st, what):
    if st != OK:
        L = load()
        raise AttambaError(f"{what}: {L.attamba_status_string(st).decode()} "
                           f"{L.attamba_last_error().decode()}".strip())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t, dtype=None, name="tensor", allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise AttambaError(f"{name} is required")
    if not t.is_cuda:
        raise AttambaError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise AttambaError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise AttambaError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise AttambaError(f"unsupported dtype {t.dtype}")


def version():
    return load().attamba_version().decode()


def uniform_chunk_count(n, P, offset):
    return int(load().attamba_uniform_chunk_count(n, P, offset))


class Index:
    """Device arrays of the compact key index (see attamba_index_t)."""

    def __init__(self, n_chunks, B, n, device="cuda", alloc=None):
        """``alloc(shape, dtype)`` returns each array (default: uninitialised device memory)."""
        if alloc is None:
            alloc = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)  # noqa: E731
        i32 = torch.int32
        self.n_chunks, self.B, self.n = int(n_chunks), int(B), int(n)
        self.cu = alloc((n_chunks + 1,), i32)
        self.bpos = alloc((n_chunks,), i32)
        self.bptr = alloc((B + 1,), i32)
        self.ls = alloc((B * n,), i32)
        self.nbb = alloc((B * n,), i32)

    def c_struct(self):
        return IndexT(self.cu.data_ptr(), self.bpos.data_ptr(), self.bptr.data_ptr(), self.ls.data_ptr(),
                      self.nbb.data_ptr(), self.n_chunks, self.B, self.n)


def chunk_index(cu_in, n_chunks, B, n, P, offset, L, mode, index, status=None, stream=None):
    st = load().attamba_chunk_index(_ptr(cu_in, torch.int32, "cu_in", allow_none=True), n_chunks, B, n, P,
                                    offset, L, mode, ctypes.byref(index.c_struct()),
                                    _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_chunk_index")


def kv_ssm_scan(x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, cu, n_chunks, K, V,
                Kc=None, Vc=None, status=None, stream=None):
    dt = x.dtype
    D = x.shape[-1]
    T = x.numel() // D
    N = A_k.shape[-1]
    f32 = torch.float32
    st = load().attamba_kv_ssm_scan(
        _dtype_code(x), _ptr(x, dt, "x"), _ptr(dt_k, dt, "dt_k"), _ptr(dt_v, dt, "dt_v"),
        _ptr(bias_k, f32, "bias_k"), _ptr(bias_v, f32, "bias_v"), _ptr(A_k, f32, "A_k"), _ptr(A_v, f32, "A_v"),
        _ptr(B_k, dt, "B_k"), _ptr(C_k, dt, "C_k"), _ptr(B_v, dt, "B_v"), _ptr(C_v, dt, "C_v"),
        _ptr(cu, torch.int32, "cu"), n_chunks, T, D, N, _ptr(K, dt, "K"), _ptr(V, dt, "V"),
        _ptr(Kc, dt, "Kc", allow_none=True), _ptr(Vc, dt, "Vc", allow_none=True),
        _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_kv_ssm_scan")


def kv_ssm_scan_u(u_k, u_v, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, cu, n_chunks, K, V,
                  Kc=None, Vc=None, status=None, stream=None):
    """attamba_kv_ssm_scan_u: the keys SSM reads u_k, the values SSM u_v (kept-projection variant)."""
    dt = u_k.dtype
    D = u_k.shape[-1]
    T = u_k.numel() // D
    N = A_k.shape[-1]
    f32 = torch.float32
    if u_v.shape != u_k.shape:
        raise AttambaError("u_k and u_v must have the same shape")
    st = load().attamba_kv_ssm_scan_u(
        _dtype_code(u_k), _ptr(u_k, dt, "u_k"), _ptr(u_v, dt, "u_v"), _ptr(dt_k, dt, "dt_k"), _ptr(dt_v, dt, "dt_v"),
        _ptr(bias_k, f32, "bias_k"), _ptr(bias_v, f32, "bias_v"), _ptr(A_k, f32, "A_k"), _ptr(A_v, f32, "A_v"),
        _ptr(B_k, dt, "B_k"), _ptr(C_k, dt, "C_k"), _ptr(B_v, dt, "B_v"), _ptr(C_v, dt, "C_v"),
        _ptr(cu, torch.int32, "cu"), n_chunks, T, D, N, _ptr(K, dt, "K"), _ptr(V, dt, "V"),
        _ptr(Kc, dt, "Kc", allow_none=True), _ptr(Vc, dt, "Vc", allow_none=True),
        _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_kv_ssm_scan_u")


def chunk_attn_fwd(q, K, V, Kc, Vc, index, scale, O, lse=None, status=None, stream=None):
    dt = q.dtype
    H, dh = q.shape[-2], q.shape[-1]
    st = load().attamba_chunk_attn_fwd(
        _dtype_code(q), _ptr(q, dt, "q"), _ptr(K, dt, "K"), _ptr(V, dt, "V"), _ptr(Kc, dt, "Kc"),
        _ptr(Vc, dt, "Vc"), ctypes.byref(index.c_struct()), H, dh, float(scale), _ptr(O, dt, "O"),
        _ptr(lse, torch.float32, "lse", allow_none=True), _ptr(status, torch.int32, "status", allow_none=True),
        _stream(stream))
    _check(st, "attamba_chunk_attn_fwd")


class Cache:
    """Device tensors of a decode cache (see attamba_cache_t)."""

    def __init__(self, state, Kb, Vb, bpos, Kr, Vr, nb, pos, P, offset):
        self.state, self.Kb, self.Vb, self.bpos, self.Kr, self.Vr, self.nb, self.pos = \
            state, Kb, Vb, bpos, Kr, Vr, nb, pos
        self.B, self.H, self.cap, self.dh = Kb.shape
        self.N = state.shape[2]
        self.L = Kr.shape[2]
        self.P, self.offset = int(P), int(offset)

    def c_struct(self):
        for name in ("state", "Kb", "Vb", "bpos", "Kr", "Vr", "nb", "pos"):
            _ptr(getattr(self, name), None, name)
        return CacheT(self.state.data_ptr(), self.Kb.data_ptr(), self.Vb.data_ptr(), self.bpos.data_ptr(),
                      self.Kr.data_ptr(), self.Vr.data_ptr(), self.nb.data_ptr(), self.pos.data_ptr(),
                      self.B, self.H, self.dh, self.N, self.P, self.offset, self.L, self.cap)


def selftest_wait_timeout(limit_ns, status, stream=None):
    """attamba_selftest_wait_timeout: a bounded wait that nothing completes; sets DEV_TIMEOUT in status."""
    L = load()
    st = L.attamba_selftest_wait_timeout(int(limit_ns), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(st, "attamba_selftest_wait_timeout")


def cache_bytes(B, H, dh, N, L, cap):
    """attamba_cache_bytes: device bytes of a bf16 decode cache with these dimensions (arrays at
    256-byte aligned offsets: state, Kb, Vb, bpos, Kr, Vr, nb, pos)."""
    c = CacheT()
    c.B, c.H, c.dh, c.N, c.L, c.cap = int(B), int(H), int(dh), int(N), int(L), int(cap)
    return int(load().attamba_cache_bytes(ctypes.byref(c)))


def decode_workspace_size(cache):
    return int(load().attamba_decode_workspace_size(ctypes.byref(cache.c_struct())))


def decode_step(cache, q_t, x_t, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, scale, o_t,
                workspace, status=None, stream=None):
    dt = torch.bfloat16
    f32 = torch.float32
    st = load().attamba_decode_step(
        BF16, ctypes.byref(cache.c_struct()), _ptr(q_t, dt, "q_t"), _ptr(x_t, dt, "x_t"),
        _ptr(dt_k, dt, "dt_k"), _ptr(dt_v, dt, "dt_v"), _ptr(bias_k, f32, "bias_k"), _ptr(bias_v, f32, "bias_v"),
        _ptr(A_k, f32, "A_k"), _ptr(A_v, f32, "A_v"), _ptr(B_k, dt, "B_k"), _ptr(C_k, dt, "C_k"),
        _ptr(B_v, dt, "B_v"), _ptr(C_v, dt, "C_v"), float(scale), _ptr(o_t, dt, "o_t"),
        _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_decode_step")


def decode_step_noalloc(cache, q_t, x_t, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, scale, o_t,
                        status=None, stream=None):
    """attamba_decode_step_noalloc: one decode step whose split-K scratch is the library's own
    fixed device array, for callers that cannot allocate a workspace (see include/attamba.h)."""
    dt = torch.bfloat16
    f32 = torch.float32
    st = load().attamba_decode_step_noalloc(
        BF16, ctypes.byref(cache.c_struct()), _ptr(q_t, dt, "q_t"), _ptr(x_t, dt, "x_t"),
        _ptr(dt_k, dt, "dt_k"), _ptr(dt_v, dt, "dt_v"), _ptr(bias_k, f32, "bias_k"), _ptr(bias_v, f32, "bias_v"),
        _ptr(A_k, f32, "A_k"), _ptr(A_v, f32, "A_v"), _ptr(B_k, dt, "B_k"), _ptr(C_k, dt, "C_k"),
        _ptr(B_v, dt, "B_v"), _ptr(C_v, dt, "C_v"), float(scale), _ptr(o_t, dt, "o_t"),
        _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_decode_step_noalloc")


def cache_from_prefill(cache, K, V, x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, n0,
                       status=None, stream=None):
    """attamba_cache_from_prefill: fill `cache` with what a prefill of positions [0, n0) of each
    sequence leaves (boundary keys/values, the last L tokens, the SSM states after n0 - 1).
    K, V: [B, n0, H, dh]; x, dt_k, dt_v: [B * n0, D]; B_k .. C_v: [B * n0, N] (bf16)."""
    dt = torch.bfloat16
    f32 = torch.float32
    st = load().attamba_cache_from_prefill(
        BF16, ctypes.byref(cache.c_struct()), _ptr(K, dt, "K"), _ptr(V, dt, "V"), _ptr(x, dt, "x"),
        _ptr(dt_k, dt, "dt_k"), _ptr(dt_v, dt, "dt_v"), _ptr(bias_k, f32, "bias_k"), _ptr(bias_v, f32, "bias_v"),
        _ptr(A_k, f32, "A_k"), _ptr(A_v, f32, "A_v"), _ptr(B_k, dt, "B_k"), _ptr(C_k, dt, "C_k"),
        _ptr(B_v, dt, "B_v"), _ptr(C_v, dt, "C_v"), int(n0),
        _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_cache_from_prefill")


def proj_gemm(X, W, outs, status=None, stream=None):
    """attamba_proj_gemm: Y = X W^T (bf16, fp32 accumulation) with Y's columns split into `outs`, a list of
    (tensor [M, width] bf16, first column) pairs in column order.  X: [M, K]; W: [Nout, K]."""
    bf = torch.bfloat16
    M, K = X.shape
    Nout = W.shape[0]
    if W.shape[1] != K:
        raise AttambaError("W must be [Nout, K] with X's K")
    segs = (ProjSegT * len(outs))()
    for k, (t, c0) in enumerate(outs):
        if t.dim() != 2 or t.shape[0] != M:
            raise AttambaError("each output must be [M, width]")
        segs[k] = ProjSegT(_ptr(t, bf, "out"), int(c0), int(t.shape[1]))
    st = load().attamba_proj_gemm(BF16, _ptr(X, bf, "X"), _ptr(W, bf, "W"), M, Nout, K, segs, len(outs),
                                  _ptr(status, torch.int32, "status", allow_none=True), _stream(stream))
    _check(st, "attamba_proj_gemm")
