"""Softmax attention over the chunk-aware key sets (oracle; test infrastructure only).

Sources
-------
* pith.science review, "What carries the argument": attention runs over the
  compressed keys/values under M_train / M_test, the map shrinking from n x n
  to about (n/P + L) x (n/P + L).
* codewithpapers.app abstract: attention is applied on the compressed
  key-value representations; W_Q (and W_O) are those of a transformer.

Readings
--------
* Scaled dot product with scale 1/sqrt(head_dim), no positional encoding, no
  dropout; head h reads channels [h*dh, (h+1)*dh) of q, K and V.
* A query whose key set is empty (only M_test with L = 0 before the first
  chunk end) returns O = 0 and LSE = -inf.
"""

import numpy as np


def masked_attention(q, k, v, mask, scale):
    """Dense n x n masked softmax attention, one sequence.

    q, k, v : [n, H, dh] (any float, computed in float64)
    mask    : [n, n] bool, mask[i, j] = query i may read key j
    Returns (O [n, H, dh], lse [H, n]) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    logits = np.einsum("ihd,jhd->hij", q, k) * scale          # [H, n, n]
    logits = np.where(mask[None, :, :], logits, -np.inf)
    m = logits.max(axis=2, keepdims=True)                      # [H, n, 1]
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(logits - m_safe)                                # exp(-inf) = 0
    l = p.sum(axis=2, keepdims=True)
    o = np.einsum("hij,jhd->ihd", p, v)
    l_safe = np.where(l > 0, l, 1.0)
    o = o / np.transpose(l_safe, (1, 0, 2))
    with np.errstate(divide="ignore"):
        lse = (m_safe + np.log(l))[:, :, 0]
    lse = np.where(empty[:, :, 0], -np.inf, lse)
    return o, lse


def attention_rows(q, k, v, rows, key_lists, scale):
    """Masked attention for selected queries only.

    rows      : list of query positions
    key_lists : for each row, the positions it attends (from mask_row)
    Returns (O [len(rows), H, dh], lse [H, len(rows)]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    H, dh = q.shape[1], q.shape[2]
    O = np.zeros((len(rows), H, dh))
    lse = np.full((H, len(rows)), -np.inf)
    for r, (i, keys) in enumerate(zip(rows, key_lists)):
        keys = np.asarray(keys, dtype=np.int64)
        if keys.size == 0:
            continue
        s = np.einsum("hd,jhd->hj", q[i], k[keys]) * scale      # [H, |S|]
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        O[r] = np.einsum("hj,jhd->hd", p, v[keys]) / l
        lse[:, r] = (m + np.log(l))[:, 0]
    return O, lse
