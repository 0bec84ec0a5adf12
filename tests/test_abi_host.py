"""Host-side checks of the C ABI (CPU only): the library loads, exports every
declared symbol, and rejects bad arguments before touching the GPU."""

import ctypes
import os
import re

import pytest

from oracle import chunks as OC
from ssm_compressed_chunked_b200 import attamba as A

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "attamba.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(attamba_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = A.load()
    names = declared_functions()
    assert set(names) == set(A.EXPORTS), names
    for name in names:
        assert hasattr(lib, name), name


def test_checked_library_exports_every_declared_symbol():
    """The bounds-checked build (ATTAMBA_CHECKED) exports the same C ABI and says so in its version."""
    path = os.path.join(os.path.dirname(A.LIB_PATH), "libattamba_checked.so")
    lib = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(lib, name), name
    lib.attamba_version.restype = ctypes.c_char_p
    assert lib.attamba_version().endswith(b"checked")


def test_version_and_status_strings():
    assert "sm_100a" in A.version()
    lib = A.load()
    assert lib.attamba_status_string(0) == b"ok"
    assert lib.attamba_status_string(1) == b"invalid argument"


@pytest.mark.parametrize("n,P,o", [(10, 4, 0), (10, 4, 3), (256, 4, 0), (2048, 4, 3), (4096, 8, 0), (1, 4, 2),
                                   (7, 1, 0), (9, 8, 7), (16, 16, 0)])
def test_uniform_chunk_count_matches_oracle_starts(n, P, o):
    assert A.uniform_chunk_count(n, P, o) == len(OC.uniform_starts(n, P, o))


def test_invalid_arguments_are_rejected_on_the_host():
    lib = A.load()
    idx = A.IndexT(0, 0, 0, 0, 0, 4, 1, 16)
    # no out arrays
    assert lib.attamba_chunk_index(None, 4, 1, 16, 4, 0, 0, 0, ctypes.byref(idx), None, None) == A.ERR_INVALID_ARG
    # wrong uniform chunk count
    fake = 1 << 20
    idx2 = A.IndexT(fake, fake, fake, fake, fake, 5, 1, 16)
    assert lib.attamba_chunk_index(None, 5, 1, 16, 4, 0, 0, 0, ctypes.byref(idx2), None, None) == A.ERR_INVALID_ARG
    # bad mode, negative L
    idx3 = A.IndexT(fake, fake, fake, fake, fake, 4, 1, 16)
    assert lib.attamba_chunk_index(None, 4, 1, 16, 4, 0, 0, 7, ctypes.byref(idx3), None, None) == A.ERR_INVALID_ARG
    assert lib.attamba_chunk_index(None, 4, 1, 16, 4, 0, -1, 0, ctypes.byref(idx3), None, None) == A.ERR_INVALID_ARG
    # scan: unsupported state size, misaligned pointer
    p = [fake] * 12
    assert lib.attamba_kv_ssm_scan(1, *p, 4, 16, 64, 24, fake, fake, None, None, None, None) == A.ERR_UNSUPPORTED
    p_bad = [fake + 2] + [fake] * 11
    assert lib.attamba_kv_ssm_scan(1, *p_bad, 4, 16, 64, 16, fake, fake, None, None, None, None) == A.ERR_INVALID_ARG
    # attention: head_dim other than 64
    assert lib.attamba_chunk_attn_fwd(1, fake, fake, fake, fake, fake, ctypes.byref(idx3), 2, 32,
                                      ctypes.c_float(0.1), fake, None, None, None) == A.ERR_UNSUPPORTED
    # decode: no leading tokens, f32 cache
    c = A.CacheT(*([fake] * 8), 1, 1, 64, 16, 8, 0, 0, 16)
    assert lib.attamba_decode_step(1, ctypes.byref(c), *([fake] * 12), ctypes.c_float(0.1), fake, fake,
                                   1 << 20, None, None) == A.ERR_INVALID_ARG
    c.L = 4
    assert lib.attamba_decode_step(0, ctypes.byref(c), *([fake] * 12), ctypes.c_float(0.1), fake, fake,
                                   1 << 20, None, None) == A.ERR_UNSUPPORTED
    assert lib.attamba_decode_workspace_size(ctypes.byref(c)) > 0
    # prefill -> cache handoff: f32, empty prefill, more boundaries than the cache holds
    c.cap = 3
    args = [fake] * 13
    assert lib.attamba_cache_from_prefill(0, ctypes.byref(c), *args, 64, None, None) == A.ERR_UNSUPPORTED
    assert lib.attamba_cache_from_prefill(1, ctypes.byref(c), *args, 0, None, None) == A.ERR_INVALID_ARG
    assert lib.attamba_cache_from_prefill(1, ctypes.byref(c), *args, 64, None, None) == A.ERR_INVALID_ARG
    assert b"exceed cap" in lib.attamba_last_error()
    # wait self-test: status word required, limit within [1 us, 1 s]
    assert lib.attamba_selftest_wait_timeout(1000000, None, None) == A.ERR_INVALID_ARG
    assert lib.attamba_selftest_wait_timeout(999, fake, None) == A.ERR_INVALID_ARG
    assert lib.attamba_selftest_wait_timeout(1000000001, fake, None) == A.ERR_INVALID_ARG


def test_empty_inputs_are_refused():
    """No sequence, no token or no chunk: every entry point rejects the call before any launch."""
    lib = A.load()
    fake = 1 << 20
    idx = A.IndexT(fake, fake, fake, fake, fake, 1, 1, 0)
    assert lib.attamba_chunk_index(None, 1, 1, 0, 4, 0, 0, 0, ctypes.byref(idx), None, None) == A.ERR_INVALID_ARG
    idx0 = A.IndexT(fake, fake, fake, fake, fake, 0, 0, 16)
    assert lib.attamba_chunk_index(None, 0, 0, 16, 4, 0, 0, 0, ctypes.byref(idx0), None, None) == A.ERR_INVALID_ARG
    assert lib.attamba_kv_ssm_scan(A.BF16, *([fake] * 12), 1, 0, 64, 16, fake, fake, None, None, None,
                                   None) == A.ERR_INVALID_ARG
    assert lib.attamba_kv_ssm_scan(A.BF16, *([fake] * 12), 0, 16, 64, 16, fake, fake, None, None, None,
                                   None) == A.ERR_INVALID_ARG
    assert lib.attamba_chunk_attn_fwd(A.BF16, fake, fake, fake, fake, fake, ctypes.byref(idx), 2, 64,
                                      ctypes.c_float(0.1), fake, None, None, None) == A.ERR_INVALID_ARG
    c = A.CacheT(*([fake] * 8), 0, 1, 64, 16, 8, 0, 4, 16)
    assert lib.attamba_decode_step(A.BF16, ctypes.byref(c), *([fake] * 12), ctypes.c_float(0.1), fake, fake,
                                   1 << 20, None, None) == A.ERR_INVALID_ARG
    assert lib.attamba_proj_gemm(A.BF16, fake, fake, 0, 64, 64, None, 0, None, None) == A.ERR_INVALID_ARG


def test_cpu_tensors_are_refused():
    import torch
    with pytest.raises(A.AttambaError):
        A._ptr(torch.zeros(4), None, "x")


@pytest.mark.parametrize("B,H,N,L,cap", [(1, 1, 16, 1, 1), (2, 16, 16, 64, 513), (3, 5, 32, 7, 33)])
def test_cache_bytes_covers_every_cache_array(B, H, N, L, cap):
    import torch
    dh = 64
    D = H * dh
    arrays = [torch.empty(2, B, N, D, dtype=torch.float32, device="meta"),
              torch.empty(B, H, cap, dh, dtype=torch.bfloat16, device="meta"),
              torch.empty(B, H, cap, dh, dtype=torch.bfloat16, device="meta"),
              torch.empty(B, cap, dtype=torch.int32, device="meta"),
              torch.empty(B, H, L, dh, dtype=torch.bfloat16, device="meta"),
              torch.empty(B, H, L, dh, dtype=torch.bfloat16, device="meta"),
              torch.empty(B, dtype=torch.int32, device="meta"),
              torch.empty(B, dtype=torch.int32, device="meta")]
    off = 0
    for t in arrays:
        assert off % 256 == 0
        off += -(-t.numel() * t.element_size() // 256) * 256
    assert A.cache_bytes(B, H, dh, N, L, cap) == off
    # degenerate dimensions give 0
    assert A.cache_bytes(B, H, 32, N, L, cap) == 0
    assert A.cache_bytes(0, H, dh, N, L, cap) == 0
    assert A.cache_bytes(B, H, dh, N, 0, cap) == 0
    assert A.cache_bytes(B, H, dh, N, L, 0) == 0


def test_layer_rejects_weights_of_the_wrong_shape_or_type():
    """layer.Layer checks every weight against the layer's sizes before it allocates anything."""
    import torch
    from ssm_compressed_chunked_b200 import layer
    B, n, D, H, dh, N = 1, 16, 128, 2, 64, 16
    bf = torch.bfloat16
    shapes = {"W_Q": (H * dh, D), "W_dtK": (D, D), "W_dtV": (D, D), "W_BK": (N, D), "W_CK": (N, D),
              "W_BV": (N, D), "W_CV": (N, D), "W_O": (D, H * dh)}
    good = {k: torch.zeros(*s, dtype=bf) for k, s in shapes.items()}
    for name in shapes:
        for bad in (torch.zeros(shapes[name][0] + 8, shapes[name][1], dtype=bf),
                    torch.zeros(*shapes[name], dtype=torch.float32)):
            w = dict(good)
            w[name] = bad
            with pytest.raises(A.AttambaError, match=name):
                layer.Layer(B, n, D, H, dh, N, w, 8, 0, 4, A.MASK_TEST, 0.125, device="cpu")
