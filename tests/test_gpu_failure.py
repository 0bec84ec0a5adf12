"""The device failure path on the GPU, without a fault: a bounded wait that nothing completes gives
up, raises ATTAMBA_DEV_TIMEOUT in the caller's status word, and leaves the context usable."""

import time

import numpy as np
import pytest
import torch

from helpers import cu_of
from ssm_compressed_chunked_b200 import attamba as A, layer, workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    A.selftest_wait_timeout(5_000_000, status)   # 5 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert status.item() == A.DEV_TIMEOUT
    assert elapsed < 2.0, elapsed   # the wait ended on its limit, far below the pipelines' 4 s

    # the context is still usable: a prefill chunk index right after matches the uniform layout
    cfg = W.shrink(W.BF16_TEST_P8_L64, B=2, n=300, D=128, H=2)
    inp = W.make_layer(cfg)
    cu = cu_of(inp)
    nch = layer.n_chunks_of(cfg, cu)
    pf = layer.Prefill(cfg.B, cfg.n, cfg.D, cfg.H, cfg.dh, cfg.N, nch, torch.bfloat16)
    pf.index_step(None, cfg.P, cfg.offset, cfg.L, layer.mode_code(cfg.mode))
    torch.cuda.synchronize()
    assert pf.status.item() == 0
    np.testing.assert_array_equal(pf.index.cu[: nch + 1].cpu().numpy(), cu)


def test_status_bits_accumulate_across_calls():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.selftest_wait_timeout(1_000_000, status)
    A.selftest_wait_timeout(1_000_000, status)
    torch.cuda.synchronize()
    assert status.item() == A.DEV_TIMEOUT   # OR-ed, not added
