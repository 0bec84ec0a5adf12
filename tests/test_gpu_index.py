"""GPU chunk index vs the oracle: bit-exact (ls, nbb, chunk ends, offsets) and the expanded mask."""

import numpy as np
import pytest
import torch

from helpers import Guarded, assert_written, chunk_starts
from oracle import chunks as OC
from oracle import mask as OM
from ssm_compressed_chunked_b200 import attamba as A
from ssm_compressed_chunked_b200 import layer
from ssm_compressed_chunked_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _gpu_index(starts_per_seq, n, L, mode, uniform=None):
    B = len(starts_per_seq)
    cu = OC.flatten_batch(starts_per_seq, n).astype(np.int32)
    nch = len(cu) - 1
    guard = Guarded()
    idx = A.Index(nch, B, n, alloc=guard)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if uniform is None:
        A.chunk_index(torch.from_numpy(cu).cuda(), nch, B, n, 1, 0, L, mode, idx, status)
    else:
        P, o = uniform
        A.chunk_index(None, nch, B, n, P, o, L, mode, idx, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    guard.check()
    for name in ("cu", "bpos", "bptr", "ls", "nbb"):
        assert_written(getattr(idx, name), name)
    return cu, idx


def _check(starts_per_seq, n, L, mode_s, idx, cu, dense=True):
    got_cu = idx.cu.cpu().numpy()
    assert np.array_equal(got_cu, cu)
    bptr = idx.bptr.cpu().numpy()
    bpos = idx.bpos.cpu().numpy()
    ls = idx.ls.cpu().numpy().reshape(len(starts_per_seq), n)
    nbb = idx.nbb.cpu().numpy().reshape(len(starts_per_seq), n)
    c0 = 0
    for b, st in enumerate(starts_per_seq):
        assert bptr[b] == c0
        rls, rnbb, rbpos = OM.compact_index(n, np.asarray(st), L, mode_s)
        assert np.array_equal(ls[b], rls), (b, "ls")
        assert np.array_equal(nbb[b], rnbb), (b, "nbb")
        assert np.array_equal(bpos[c0:c0 + len(st)], rbpos), (b, "bpos")
        if dense:
            exp = OM.expand_compact(n, ls[b], nbb[b], bpos[c0:c0 + len(st)])
            assert np.array_equal(exp, OM.dense_mask(n, np.asarray(st), L, mode_s)), b
        c0 += len(st)
    assert bptr[len(starts_per_seq)] == c0


def test_random_sweep():
    rng = np.random.default_rng(2024)
    for case in range(150):
        B = int(rng.integers(1, 4))
        n = int(rng.integers(1, 90))
        L = int(rng.integers(0, n + 3))
        mode_s = OM.MODES[int(rng.integers(2))]
        mode = layer.mode_code(mode_s)
        kind = case % 3
        if kind == 2:
            starts = [OC.varlen_starts(rng.integers(1, 12, size=n + 1).tolist(), n) for _ in range(B)]
            cu, idx = _gpu_index(starts, n, L, mode)
        else:
            P = int(rng.integers(1, 9))
            o = int(rng.integers(0, P)) if kind == 1 else 0
            starts = [OC.uniform_starts(n, P, o)] * B
            cu, idx = _gpu_index(starts, n, L, mode, uniform=(P, o))
        _check(starts, n, L, mode_s, idx, cu)


@pytest.mark.parametrize("cfg", W.LAYER_CONFIGS, ids=lambda c: c.name)
def test_configs(cfg):
    starts = chunk_starts(W.make_layer(cfg))
    uniform = None if cfg.varlen is not None else (cfg.P, cfg.offset)
    cu, idx = _gpu_index(starts, cfg.n, cfg.L, layer.mode_code(cfg.mode), uniform)
    _check(starts, cfg.n, cfg.L, cfg.mode, idx, cu, dense=cfg.n <= 2048)


def test_malformed_offsets_raise_the_status_bit():
    n, B = 32, 2
    cu = np.array([0, 5, 3, 40, 64], dtype=np.int32)  # not increasing, and a chunk crosses position 32
    idx = A.Index(4, B, n)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.chunk_index(torch.from_numpy(cu).cuda(), 4, B, n, 1, 0, 2, A.MASK_TRAIN, idx, status)
    torch.cuda.synchronize()
    assert status.item() & A.DEV_BAD_CHUNKS
