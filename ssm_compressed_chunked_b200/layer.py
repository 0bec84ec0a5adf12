"""The prefill hot path as three C-ABI calls on preallocated device buffers,
and the whole layer with its projections around it.

    chunk_index  ->  kv_ssm_scan (K and V, plus the chunk-end rows Kc, Vc)  ->  chunk_attn_fwd

    Layer:  x  --proj_gemm-->  q, dt_K, dt_V, B_K, C_K, B_V, C_V  --hot path-->  O  --proj_gemm-->  y = O W_O

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


# the layer's input projections, in the column order of the one GEMM that computes them
INPUT_PROJECTIONS = ("W_Q", "W_dtK", "W_dtV", "W_BK", "W_CK", "W_BV", "W_CV")


class Layer:
    """One Attamba layer forward, y = Attn(q, K, V) W_O, on preallocated device buffers.

    pith.science review of Attamba, "Core claim": the keys and values come from
    two SSMs over the layer input (K = SSM_K(x), V = SSM_V(x)) in place of W_K
    and W_V, while the query and output projections stay; "Assumptions & free
    parameters": each SSM is Mamba's selective SSM, whose step and B, C are
    projections of its input.  So x is projected seven ways (q, dt_K, dt_V, B_K,
    C_K, B_V, C_V) by one GEMM whose column segments land in the arrays the hot
    path reads, the hot path gives O, and a second GEMM gives y = O W_O.

    ``weights`` maps each name of INPUT_PROJECTIONS and "W_O" to a bf16 matrix in
    [out, in] layout (W_Q [H dh, D]; W_dtK, W_dtV [D, D]; W_BK ... W_CV [N, D];
    W_O [D, H dh]) and "bias_k", "bias_v" [D], "A_k", "A_v" [D, N] to fp32; all on
    the layer's device.  The chunking is uniform (P, offset) unless ``forward``
    gets chunk offsets ``cu_in`` (then ``n_chunks`` must be their count);
    ``mode`` is MASK_TEST or MASK_TRAIN.

    Decoding (pith.science review, "Core claim": the inference cache holds the
    chunk boundary states, and "If this is right": P = 8 with 64 leading tokens)
    continues a uniform-chunk prefill one token at a time under M_test:
    ``new_cache`` or ``cache_from_prefill`` gives the cache, ``decode_step`` maps
    x_t to y_t."""

    def __init__(self, B, n, D, H, dh, N, weights, P, offset, L, mode, scale, n_chunks=None, device="cuda",
                 alloc=None):
        bf = torch.bfloat16
        self.B, self.n, self.D, self.H, self.dh, self.N = B, n, D, H, dh, N
        self.P, self.offset, self.L, self.mode, self.scale = P, offset, L, mode, scale
        T = B * n
        shapes = {"W_Q": (H * dh, D), "W_dtK": (D, D), "W_dtV": (D, D), "W_BK": (N, D), "W_CK": (N, D),
                  "W_BV": (N, D), "W_CV": (N, D), "W_O": (D, H * dh)}
        for name, shape in shapes.items():
            w = weights[name]
            if tuple(w.shape) != shape or w.dtype != bf:
                raise A.AttambaError(f"{name} must be bf16 {shape}, got {w.dtype} {tuple(w.shape)}")
        self.W_in = torch.cat([weights[k] for k in INPUT_PROJECTIONS], dim=0).contiguous()
        self.W_O = weights["W_O"].contiguous()
        self.bias_k, self.bias_v = weights["bias_k"], weights["bias_v"]
        self.A_k, self.A_v = weights["A_k"], weights["A_v"]
        if alloc is None:
            alloc = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)  # noqa: E731
        widths = [shapes[k][0] for k in INPUT_PROJECTIONS]
        self.proj, c = [], 0
        for w in widths:
            self.proj.append((alloc((T, w), bf), c))
            c += w
        if n_chunks is None:
            n_chunks = B * A.uniform_chunk_count(n, P, offset)
        self.prefill = Prefill(B, n, D, H, dh, N, n_chunks, bf, device=device, alloc=alloc)
        self.y = alloc((T, D), bf)
        self.status = self.prefill.status
        self._step = None   # decode buffers, made by the first decode_step

    @property
    def projections(self):
        """The projected activations, by the names of INPUT_PROJECTIONS without the "W_"."""
        return {k[2:]: t for k, (t, _) in zip(INPUT_PROJECTIONS, self.proj)}

    # ---------------------------------------------------------------- decode (M_test, uniform chunks)
    def new_cache(self, cap, device=None):
        """An empty decode cache (every sequence at position 0) with room for ``cap`` chunk-end rows
        per sequence and the layer's L most recent tokens, chunked like the layer (P, offset); on the
        layer's device unless ``device`` says otherwise."""
        if self.L < 1:
            raise A.AttambaError("decoding keeps the L >= 1 most recent tokens; this layer has L = 0")
        device = self.W_in.device if device is None else device
        B, H, dh, N, D, L = self.B, self.H, self.dh, self.N, self.D, self.L
        bf, i32 = torch.bfloat16, torch.int32
        z = lambda *shape, dt=bf: torch.zeros(*shape, dtype=dt, device=device)  # noqa: E731
        return A.Cache(z(2, B, N, D, dt=torch.float32), z(B, H, cap, dh), z(B, H, cap, dh), z(B, cap, dt=i32),
                       z(B, H, L, dh), z(B, H, L, dh), z(B, dt=i32), z(B, dt=i32), self.P, self.offset)

    def cache_from_prefill(self, cache, x, stream=None):
        """Fill ``cache`` with what the last ``forward`` (over x, all n tokens of each sequence, uniform
        chunks) leaves for decoding position n onwards: its chunk-end keys and values, its last L
        tokens and the SSM states after token n - 1."""
        B, n, H, dh = self.B, self.n, self.H, self.dh
        pf = self.prefill
        _, dt_k, dt_v, B_k, C_k, B_v, C_v = (t for t, _ in self.proj)
        A.cache_from_prefill(cache, pf.K.view(B, n, H, dh), pf.V.view(B, n, H, dh), x, dt_k, dt_v, self.bias_k,
                             self.bias_v, self.A_k, self.A_v, B_k, C_k, B_v, C_v, n, self.status, stream)

    def decode_step(self, cache, x_t, stream=None):
        """One new token per sequence under the inference mask M_test: x_t [B, D] bf16 -> y_t [B, D]
        (the layer's own buffer).  The same seven projections as ``forward`` (one GEMM of B rows), the
        decode step over ``cache`` (which it advances by one position), then W_O."""
        B, H, dh, D = self.B, self.H, self.dh, self.D
        bf = torch.bfloat16
        if self._step is None:
            dev = self.W_in.device
            self._step, c = [], 0
            for (t, _) in self.proj:
                self._step.append((torch.empty(B, t.shape[1], dtype=bf, device=dev), c))
                c += t.shape[1]
            self.o_t = torch.empty(B, H, dh, dtype=bf, device=dev)
            self.y_t = torch.empty(B, D, dtype=bf, device=dev)
            self._ws = {}
        size = A.decode_workspace_size(cache)
        if size not in self._ws:
            self._ws[size] = torch.empty(size, dtype=torch.uint8, device=self.W_in.device)
        q, dt_k, dt_v, B_k, C_k, B_v, C_v = (t for t, _ in self._step)
        A.proj_gemm(x_t, self.W_in, self._step, self.status, stream)
        A.decode_step(cache, q.view(B, H, dh), x_t, dt_k, dt_v, self.bias_k, self.bias_v, self.A_k, self.A_v, B_k,
                      C_k, B_v, C_v, self.scale, self.o_t, self._ws[size], self.status, stream)
        A.proj_gemm(self.o_t.view(B, H * dh), self.W_O, [(self.y_t, 0)], self.status, stream)
        return self.y_t

    @property
    def step_projections(self):
        """The last decode step's projections, named like ``projections``."""
        if self._step is None:
            raise A.AttambaError("no decode step has run on this layer")
        return {k[2:]: t for k, (t, _) in zip(INPUT_PROJECTIONS, self._step)}

    def forward(self, x, cu_in=None, stream=None):
        """x [B n, D] bf16 -> y [B n, D] bf16 (the layer's own buffer)."""
        T, H, dh = self.B * self.n, self.H, self.dh
        q, dt_k, dt_v, B_k, C_k, B_v, C_v = (t for t, _ in self.proj)
        A.proj_gemm(x, self.W_in, self.proj, self.status, stream)
        pf = self.prefill
        pf.index_step(cu_in, self.P if cu_in is None else 1, self.offset, self.L, self.mode, stream)
        pf.scan_step(x, dt_k, dt_v, self.bias_k, self.bias_v, self.A_k, self.A_v, B_k, C_k, B_v, C_v, stream)
        pf.attn_step(q.view(T, H, dh), self.scale, stream)
        A.proj_gemm(pf.O.view(T, H * dh), self.W_O, [(self.y, 0)], self.status, stream)
        return self.y

