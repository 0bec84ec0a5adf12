"""attamba_decode_step_noalloc against attamba_decode_step (GPU).

The no-alloc entry point serves callers that cannot hand the library a device
workspace at decode time (a host that pre-sizes all device memory and forbids
allocation once it is serving, or a caller with no way to pass a scratch
buffer): it keeps its split-K partials in a fixed array inside the library.
This file runs after every other test file (pytest collects it last).
"""

import ctypes

import pytest
import torch

from decode_cases import decode_from_empty_vs_oracle, handoff_then_decode
from helpers import BF16_ATOL, assert_written, decode_cache_contents, gpu_cache, poison_
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_noalloc_step_matches_the_workspace_step_on_two_calls_in_a_row():
    cfg = W.DECODE_CONFIG
    dec = W.make_decode(cfg)
    contents = decode_cache_contents(dec)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in dec.items()}
    ref = gpu_cache(contents, cfg.P, cfg.offset)
    new = gpu_cache(contents, cfg.P, cfg.offset)
    assert A.decode_workspace_size(ref) <= 4 << 20
    ws = torch.empty(A.decode_workspace_size(ref), dtype=torch.uint8, device="cuda")
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    st_new = torch.zeros(1, dtype=torch.int32, device="cuda")
    for s in range(2):
        args = (g["q"][s], g["x"][s], g["dt_k"][s], g["dt_v"][s], g["bias_k"], g["bias_v"], g["A_k"], g["A_v"],
                g["B_k"][s], g["C_k"][s], g["B_v"][s], g["C_v"][s], dec["scale"])
        o_ref = poison_(torch.empty(cfg.B, cfg.H, cfg.dh, dtype=torch.bfloat16, device="cuda"))
        o_new = poison_(torch.empty_like(o_ref))
        A.decode_step(ref, *args, o_ref, ws, st_ref)
        A.decode_step_noalloc(new, *args, o_new, st_new)
        torch.cuda.synchronize()
        assert_written(o_ref, "o_t (workspace step)")
        assert_written(o_new, "o_t (no-alloc step)")
        err = (o_new.float() - o_ref.float()).abs().max().item()
        assert err <= BF16_ATOL, (s, err)
    assert st_ref.item() == 0 and st_new.item() == 0
    # the caches advanced identically (rows no step has written yet hold NaN in both)
    for name in ("state", "Kr", "Vr", "Kb", "Vb", "bpos", "nb", "pos"):
        a, b = getattr(ref, name), getattr(new, name)
        if a.is_floating_point():
            assert torch.equal(a.isnan(), b.isnan()), name
            a, b = a.nan_to_num(0.0), b.nan_to_num(0.0)
        assert torch.equal(a, b), name


def test_noalloc_decode_from_empty_cache_at_workload_size_matches_oracle():
    """The no-alloc step from an empty cache at the decode workload's dimensions (two splits per
    sequence and head, one of them without keys at the first step) against the oracle's decode."""
    decode_from_empty_vs_oracle(W.shrink(W.DECODE_CONFIG, seed=41), 24, noalloc=True)


def test_noalloc_decode_after_short_handoff_matches_oracle():
    """The no-alloc step after a 100-token prefill handed into a cache of capacity 2064 (16 splits over
    about 70 keys) against the oracle's scan, handoff and decode."""
    handoff_then_decode(100, 24, 2064, noalloc=True)


def test_noalloc_step_rejects_a_cache_beyond_its_scratch():
    lib = A.load()
    fake = 1 << 20  # never dereferenced: the size check comes before any launch
    c = A.CacheT(*([fake] * 8), 128, 128, 64, 16, 8, 0, 64, 16)   # 128 x 128 heads need more than 4 MiB
    assert lib.attamba_decode_workspace_size(ctypes.byref(c)) > 4 << 20
    st = lib.attamba_decode_step_noalloc(A.BF16, ctypes.byref(c), *([fake] * 12), ctypes.c_float(0.125), fake,
                                         None, None)
    assert st == A.ERR_UNSUPPORTED
    assert b"scratch" in lib.attamba_last_error()
