"""The prefill hot path as three C-ABI calls on preallocated device buffers.

    chunk_index  ->  kv_ssm_scan (K and V, plus the chunk-end rows Kc, Vc)  ->  chunk_attn_fwd

Only buffer allocation happens here (torch, once); every step of the path runs
in libattamba.so.
"""

import torch

from . import attamba as A


class Prefill:
    """Device buffers of one prefill and the three calls over them.

    ``alloc(shape, dtype)`` returns each output buffer (default: uninitialised
    device memory); a caller can hand in its own, e.g. pre-filled memory."""

    def __init__(self, B, n, D, H, dh, N, n_chunks, dtype, device="cuda", alloc=None):
        self.B, self.n, self.D, self.H, self.dh, self.N = B, n, D, H, dh, N
        self.n_chunks = n_chunks
        self.dtype = dtype
        T = B * n
        if alloc is None:
            alloc = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)  # noqa: E731
        self.index = A.Index(n_chunks, B, n, device, alloc=alloc)
        self.K = alloc((T, D), dtype)
        self.V = alloc((T, D), dtype)
        self.Kc = alloc((n_chunks, D), dtype)
        self.Vc = alloc((n_chunks, D), dtype)
        self.O = alloc((T, H, dh), dtype)
        self.lse = alloc((B, H, n), torch.float32)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def index_step(self, cu_in, P, offset, L, mode, stream=None):
        A.chunk_index(cu_in, self.n_chunks, self.B, self.n, P, offset, L, mode, self.index, self.status, stream)

    def scan_step(self, x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, stream=None):
        A.kv_ssm_scan(x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, self.index.cu,
                      self.n_chunks, self.K, self.V, self.Kc, self.Vc, self.status, stream)

    def attn_step(self, q, scale, stream=None):
        H, dh = self.H, self.dh
        A.chunk_attn_fwd(q, self.K.view(-1, H, dh), self.V.view(-1, H, dh), self.Kc.view(-1, H, dh),
                         self.Vc.view(-1, H, dh), self.index, scale, self.O, self.lse, self.status, stream)

    def forward(self, x, q, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, cu_in, P, offset, L,
                mode, scale, stream=None):
        self.index_step(cu_in, P, offset, L, mode, stream)
        self.scan_step(x, dt_k, dt_v, bias_k, bias_v, A_k, A_v, B_k, C_k, B_v, C_v, stream)
        self.attn_step(q, scale, stream)
        return self.O


def n_chunks_of(cfg, cu=None):
    """Chunk count of a workload: uniform from the library's count, variable from its cu array."""
    if cfg.varlen is None:
        return cfg.B * A.uniform_chunk_count(cfg.n, cfg.P, cfg.offset)
    return len(cu) - 1


def mode_code(mode):
    return A.MASK_TRAIN if mode == "train" else A.MASK_TEST
