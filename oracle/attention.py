"""O1 -- masked (block-sparse) softmax attention, float64, CPU.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Definition followed (CalibAtt paper page, Abstract and Figure 5(b) top: the
kept connections are computed exactly, the unset blocks are skipped).  For
batch b, head h and a real query row i < N in query block qb = i // Bq:

    J(i)   = { j < N : mask[h, qb, j // Bk] = 1 }
    s_ij   = scale * <q_i, k_j>              for j in J(i)
    m_i    = max_j s_ij
    O_i    = sum_j exp(s_ij - m_i) v_j / sum_j exp(s_ij - m_i)
    LSE_i  = m_i + log sum_j exp(s_ij - m_i)

A row with J(i) empty, and every padded row i >= N, gets O_i = 0 and
LSE_i = -inf.  The mask is shared across the batch.  ``scale`` is the exact
value the kernel multiplies by (the float32 of 1/sqrt(d) by default), passed in
so both sides use the same number.

The computation is blockwise only in the sense the definition already is: one
query block at a time against the concatenation of its kept key blocks, with a
numpy matmul as the dot-product step.
"""

from __future__ import annotations

import numpy as np


def _as_f64(x):
    return np.asarray(x, dtype=np.float64)


def _kept_keys(mask_row, N, block_k):
    """Token indices j < N of the key blocks marked 1 in ``mask_row``."""
    kbs = np.nonzero(np.asarray(mask_row))[0]
    if kbs.size == 0:
        return np.zeros(0, dtype=np.int64)
    idx = (kbs[:, None] * block_k + np.arange(block_k)[None, :]).reshape(-1)
    return idx[idx < N]


def _attend_rows(q_rows, k_h, v_h, keys, scale):
    """Softmax attention of ``q_rows`` over the key tokens ``keys``."""
    n_rows, d = q_rows.shape
    if keys.size == 0 or n_rows == 0:
        return np.zeros((n_rows, v_h.shape[1])), np.full(n_rows, -np.inf)
    s = scale * (q_rows @ k_h[keys].T)
    m = s.max(axis=1)
    p = np.exp(s - m[:, None])
    l = p.sum(axis=1)
    o = (p @ v_h[keys]) / l[:, None]
    lse = m + np.log(l)
    return o, lse


def masked_attention_rows(q, k, v, mask, N, block_q, block_k, scale, b, h, qb):
    """O and LSE for the rows of one query block ``qb`` of (batch b, head h).

    ``q, k, v``: [B, H, Np, d]; ``mask``: [H, nqb, nkb] (already the slice of
    the mask dictionary for these heads).  Returns (O [Bq, d], LSE [Bq]) for
    rows qb*Bq .. qb*Bq+Bq-1; rows >= N are 0 / -inf.
    """
    q = _as_f64(q[b, h])
    k = _as_f64(k[b, h])
    v = _as_f64(v[b, h])
    scale = float(np.float64(scale))
    r0 = qb * block_q
    r1 = r0 + block_q
    o = np.zeros((block_q, v.shape[1]))
    lse = np.full(block_q, -np.inf)
    real = min(r1, N) - r0
    if real > 0:
        keys = _kept_keys(mask[h, qb], N, block_k)
        o_r, lse_r = _attend_rows(q[r0:r0 + real], k, v, keys, scale)
        o[:real] = o_r
        lse[:real] = lse_r
    return o, lse


def masked_attention(q, k, v, mask, N, block_q, block_k, scale):
    """Full O1 over every (b, h, query block).  Returns (O, LSE) in float64.

    ``q, k, v``: [B, H, Np, d] (any float dtype, read exactly);
    ``mask``: [H, nqb, nkb] with nqb = Np / Bq, nkb = Np / Bk.
    """
    q = _as_f64(q)
    B, H, Np, d = q.shape
    dv = np.shape(v)[3]
    nqb = Np // block_q
    mask = np.asarray(mask)
    assert mask.shape[0] == H and mask.shape[1] == nqb and mask.shape[2] == Np // block_k
    O = np.zeros((B, H, Np, dv))
    LSE = np.full((B, H, Np), -np.inf)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                o, lse = masked_attention_rows(q, k, v, mask, N, block_q, block_k, scale, b, h, qb)
                O[b, h, qb * block_q:(qb + 1) * block_q] = o
                LSE[b, h, qb * block_q:(qb + 1) * block_q] = lse
    return O, LSE

