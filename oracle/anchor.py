"""O8 -- spatial repetition: anchor query rows and broadcast.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The paper page observes that attention maps repeat across the spatial rows of
a frame (Figure 4), computes attention for only k anchor query rows per frame
and broadcasts their outputs to the neighbouring rows (Figure 5(b) bottom),
and times attention restricted to k of the 30 spatial rows per frame at 480p
(Table S4: k = 15, 10, 5, 4, 3 gives 50 ... 90% row sparsity).  Readings
taken: the k anchor rows are evenly spaced and centred in the frame (row
floor((i + 1/2) * rows / k) for i < k); every row takes the output of its
nearest anchor row (the lower one on a tie), in the same frame and column;
anchor queries attend to every real key.  Head selection by a spatial
similarity score (Figure S13, tau = 0.87) is left to the caller.
"""

from __future__ import annotations

import math

import numpy as np


def anchor_rows(rows, k):
    """(anchor rows, nearest anchor of every row)."""
    anchors = []
    for i in range(k):
        anchors.append(int(math.floor((i + 0.5) * rows / k)))
    nearest = []
    for r in range(rows):
        best = None
        for a in anchors:
            if best is None or abs(a - r) < abs(best - r) or (abs(a - r) == abs(best - r) and a < best):
                best = a
        nearest.append(best)
    return anchors, nearest


def anchor_attention(q, k, v, N, frames, rows, cols, k_anchor, scale):
    """O [B, H, Np, d] float64: softmax(scale q_a K^T) V of each token's anchor token a, over the real keys."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, Np, d = q.shape
    _, nearest = anchor_rows(rows, k_anchor)
    out = np.zeros((B, H, Np, d))
    for b in range(B):
        for h in range(H):
            cache = {}
            for t in range(N):
                f, rem = divmod(t, rows * cols)
                r, c = divmod(rem, cols)
                ta = f * rows * cols + nearest[r] * cols + c
                if ta not in cache:
                    s = scale * (k[b, h, :N] @ q[b, h, ta])
                    p = np.exp(s - s.max())
                    cache[ta] = (p @ v[b, h, :N]) / p.sum()
                out[b, h, t] = cache[ta]
    return out


def anchor_attention_tokens(q, k, v, N, frames, rows, cols, k_anchor, scale, b, h, tokens):
    """O8 for selected tokens of (batch b, head h): [len(tokens), d] float64.

    Token t takes softmax(scale q_a K^T) V of its anchor token a (same frame
    and column, nearest anchor row) over the real keys; for full-size inputs,
    where computing every token is too slow.
    """
    kh = np.asarray(k[b, h, :N], np.float64)
    vh = np.asarray(v[b, h, :N], np.float64)
    _, nearest = anchor_rows(rows, k_anchor)
    out = np.zeros((len(tokens), vh.shape[1]))
    for i, t in enumerate(tokens):
        if t >= N:
            continue
        f, rem = divmod(int(t), rows * cols)
        r, c = divmod(rem, cols)
        ta = f * rows * cols + nearest[r] * cols + c
        s = scale * (kh @ np.asarray(q[b, h, ta], np.float64))
        p = np.exp(s - s.max())
        out[i] = (p @ vh) / p.sum()
    return out
