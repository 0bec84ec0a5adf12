"""Token-by-token decode over the boundary-state cache (oracle; test infrastructure only).

Sources
-------
* pith.science review, "Core claim": at inference only the boundary states are
  cached, so the KV cache and the attention map shrink by a factor of P.
* pith.science review, "If this is right": only the final SSM state of each
  chunk is cached; P = 8 with 64 leading tokens gives about 8x compression.
* pith.science review, "What carries the argument": M_test (Eq. 7) with the
  leading-token window (Eq. 8).
* pith.science review, Referee Report, major comment on Eq. (7): only completed
  chunks are attended; the current chunk is reached through the leading tokens.

Readings
--------
* Chunks are uniform with size P and offset o = offset mod P.  Position t
  starts a chunk when t == 0 or (t >= o and (t - o) mod P == 0) and ends one
  when t + 1 starts one.  (The sequence has no fixed end during decode.)
* A step at position t: reset the SSM state if t starts a chunk, apply the
  same update as the prefill scan, emit k_t and v_t, keep them among the L most
  recent tokens, and, if t ends a chunk, append them to the boundary list.
  The query then attends the boundaries at positions < t - L + 1 together with
  the window [t - L + 1, t].  L must be at least 1.
"""

import numpy as np

from .ssm import softplus


def is_chunk_start(t, P, offset):
    o = offset % P
    return t == 0 or (t >= o and (t - o) % P == 0)


def is_chunk_end(t, P, offset):
    return is_chunk_start(t + 1, P, offset) and t + 1 > 0


class DecodeCache:
    """Cache of one batch, everything in float64.

    state[s]   : [B, D, N] SSM state of s in (0 = keys, 1 = values)
    bpos[b]    : list of boundary positions, increasing
    Kb[b],Vb[b]: lists of [H, dh] boundary keys / values
    ring[b]    : dict position -> (k [H, dh], v [H, dh]) for the last L positions
    pos[b]     : next position to decode
    """

    def __init__(self, B, H, dh, N, P, offset, L):
        if L < 1:
            raise ValueError("decode needs at least one leading token (L >= 1)")
        self.B, self.H, self.dh, self.N = B, H, dh, N
        self.P, self.offset, self.L = P, offset, L
        D = H * dh
        self.state = np.zeros((2, B, D, N))
        self.bpos = [[] for _ in range(B)]
        self.Kb = [[] for _ in range(B)]
        self.Vb = [[] for _ in range(B)]
        self.ring = [dict() for _ in range(B)]
        self.pos = [0] * B

    def step(self, q, x, dt, dt_bias, A, Bm, Cm, scale):
        """One decode step for every sequence.

        q       : [B, H, dh]
        x       : [B, D]
        dt      : [2, B, D]   pre-softplus steps of the key and value SSMs
        dt_bias : [2, D]
        A       : [2, D, N]
        Bm, Cm  : [2, B, N]
        Returns o [B, H, dh] float64.
        """
        B, H, dh, L = self.B, self.H, self.dh, self.L
        out = np.zeros((B, H, dh))
        for b in range(B):
            t = self.pos[b]
            kv = []
            for s in range(2):
                delta = softplus(np.asarray(dt[s][b], np.float64) + np.asarray(dt_bias[s], np.float64))
                h = self.state[s, b]
                if is_chunk_start(t, self.P, self.offset):
                    h = np.zeros_like(h)
                h = (np.exp(delta[:, None] * np.asarray(A[s], np.float64)) * h
                     + (delta * np.asarray(x[b], np.float64))[:, None] * np.asarray(Bm[s][b], np.float64)[None, :])
                self.state[s, b] = h
                kv.append((h @ np.asarray(Cm[s][b], np.float64)).reshape(H, dh))
            k_t, v_t = kv
            self.ring[b][t] = (k_t, v_t)
            for p in [p for p in self.ring[b] if p <= t - L]:
                del self.ring[b][p]
            if is_chunk_end(t, self.P, self.offset):
                self.bpos[b].append(t)
                self.Kb[b].append(k_t)
                self.Vb[b].append(v_t)
            lo = max(0, t - L + 1)
            keys, vals = [], []
            for p, kk, vv in zip(self.bpos[b], self.Kb[b], self.Vb[b]):
                if p < lo:
                    keys.append(kk)
                    vals.append(vv)
            for p in range(lo, t + 1):
                kk, vv = self.ring[b][p]
                keys.append(kk)
                vals.append(vv)
            Kx = np.stack(keys, axis=1)                 # [H, nk, dh]
            Vx = np.stack(vals, axis=1)
            qb = np.asarray(q[b], np.float64)
            s_ = np.einsum("hd,hjd->hj", qb, Kx) * scale
            m = s_.max(axis=1, keepdims=True)
            p_ = np.exp(s_ - m)
            out[b] = np.einsum("hj,hjd->hd", p_, Vx) / p_.sum(axis=1, keepdims=True)
            self.pos[b] = t + 1
        return out

    def n_keys(self, b, t):
        """|S_test(t)| for a query at position t of sequence b (boundaries below the window + window)."""
        lo = max(0, t - self.L + 1)
        return sum(1 for p in self.bpos[b] if p < lo) + (t + 1 - lo)


def cache_from_prefill(K, V, h_last, n0, P, offset, L, H, dh, N):
    """Cache that a prefill of positions [0, n0) leaves behind, one sequence per batch row.

    K, V   : [B, n0, H, dh] prefill keys / values (uniform chunks P, offset)
    h_last : [2, B, D, N] SSM states after position n0 - 1
    Boundaries are the positions < n0 that end a chunk under the uniform rule
    (the prefill's cut of the last chunk at n0 - 1 is not a chunk end here).
    """
    B = K.shape[0]
    c = DecodeCache(B, H, dh, N, P, offset, L)
    c.state = np.array(h_last, dtype=np.float64)
    for b in range(B):
        for p in range(n0):
            if is_chunk_end(p, P, offset):
                c.bpos[b].append(p)
                c.Kb[b].append(np.asarray(K[b, p], np.float64))
                c.Vb[b].append(np.asarray(V[b, p], np.float64))
        for p in range(max(0, n0 - L), n0):
            c.ring[b][p] = (np.asarray(K[b, p], np.float64), np.asarray(V[b, p], np.float64))
        c.pos[b] = n0
    return c
