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
anchor queries attend to every real key.

O9 -- the spatial-similarity score and the repetition dictionary.  Figure
5(a) flags the heads whose maps repeat across spatial rows; Figure 6(a)
plots each map's "spatial similarity" and Figure S13 flags heads whose score
exceeds tau = 0.87, but the pages do not define the score.  Reading taken:
the mean, over the video query tokens (f, r, c) with r < rows - 1, of the
cosine similarity of the dense attention rows (softmax over all real keys)
of (f, r, c) and (f, r + 1, c); the dictionary flags a map when its score,
averaged over the calibration inputs, is at least tau.
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


def spatial_similarity(q, k, N, frames, rows, cols, scale):
    """O9: score [H] float64 of one input; ``q, k``: [H, Np, d].

    Video token t = (f rows + r) cols + c for t < frames rows cols; real
    tokens beyond (text) are keys only.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    H = q.shape[0]
    fr = rows * cols
    out = np.zeros(H)
    for h in range(H):
        kh = k[h, :N]
        total, count = 0.0, 0
        for f in range(frames):
            s = scale * (q[h, f * fr:(f + 1) * fr] @ kh.T)    # the frame's query rows against every real key
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            a = p[:(rows - 1) * cols]                        # rows r < rows - 1 ...
            b = p[cols:]                                     # ... and the row below, same column
            cos = (a * b).sum(axis=1) / np.sqrt((a * a).sum(axis=1) * (b * b).sum(axis=1))
            total += cos.sum()
            count += cos.size
        out[h] = total / count
    return out


def repetition_flags(scores, tau):
    """Repetition dictionary from per-input scores [n_inputs, n_maps]: (mean, flags).

    The mean is taken the way the GPU takes it, a float32 sum in input order
    divided by the input count, so the flag decision (mean >= tau, float32)
    is made in the same precision on both sides.
    """
    scores = np.asarray(scores, np.float32)
    acc = np.zeros(scores.shape[1], np.float32)
    for i in range(scores.shape[0]):
        acc = (acc + scores[i]).astype(np.float32)
    mean = (acc / np.float32(scores.shape[0])).astype(np.float32)
    return mean, (mean >= np.float32(tau)).astype(np.uint8)
