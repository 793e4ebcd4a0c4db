"""O2-O4 -- calibration: block energy, per-row selection, agreement voting.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Steps, in the order the CalibAtt paper page gives them (Figure 5(a): threshold
the top key blocks per query block, then aggregate the resulting masks across
prompts into a mask dictionary):

1. ``block_energy`` -- the block-level post-softmax attention map (Figure 2,
   "token-level or block-level" post-softmax maps; Table S5 calls the
   quantities "block energies").  Reading taken: E[qb, kb] is the mean, over
   the real query rows of block qb, of the dense softmax probability mass that
   falls on the real keys of block kb.  No mask is applied while scoring.
   Every E row therefore sums to 1.
2. ``select_topk`` -- keep the k key blocks with the largest energy, ties to
   the smaller key-block index; k = min(nkb, max(1, ceil(frac * nkb))).
   ``select_energy`` -- keep the shortest prefix of that same order whose
   running float64 sum reaches (1 - eps) * (float64 sum of the row in key-block
   order); the block that crosses the threshold is kept (Figure S8 names an
   energy threshold eps but prints no values).
3. ``vote`` -- votes = number of inputs that kept the block (Figure 3(b):
   keep frequency 0 = always skipped, 1 = always computed); keep iff
   votes >= min_votes with min_votes = ceil(rho * I) (Figure 7: agreement
   threshold rho).  A query-block row left empty by the vote keeps exactly one
   key block: the one with the most votes, then the largest float32 energy
   sum (accumulated in input order, the precision the GPU uses for this
   integer decision), then the smallest index.
"""

from __future__ import annotations

import math

import numpy as np


def _energy_row(q_rows, k_real, N, block_k, nkb, scale):
    """E[qb, :] of one query block: its real rows ``q_rows`` against the real keys."""
    s = scale * (q_rows @ k_real.T)              # [rows, N] dense scores
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p /= p.sum(axis=1, keepdims=True)            # dense softmax rows
    col_mass = p.sum(axis=0)                     # summed over the block's rows
    row = np.zeros(nkb)
    for kb in range(nkb):
        c0, c1 = kb * block_k, min((kb + 1) * block_k, N)
        if c1 > c0:
            row[kb] = col_mass[c0:c1].sum() / q_rows.shape[0]
    return row


def block_energy(q, k, N, block_q, block_k, scale):
    """Block energies of one calibration input.

    ``q, k``: [H, Np, d] (any float dtype, read exactly).  Returns
    E [H, nqb, nkb] float64 with nkb = ceil(N / block_k): the key grid covers
    the real keys only (Table S6 varies the key-block size independently of
    the query block, and a key block past the sequence would hold no key).
    Padded query rows (>= N) are excluded from the mean.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    H, Np, d = q.shape
    nqb, nkb = Np // block_q, -(-N // block_k)
    scale = float(np.float64(scale))
    E = np.zeros((H, nqb, nkb))
    for h in range(H):
        kh = k[h, :N]
        for qb in range(nqb):
            r0 = qb * block_q
            r1 = min(r0 + block_q, N)
            if r1 <= r0:
                continue
            E[h, qb] = _energy_row(q[h, r0:r1], kh, N, block_k, nkb, scale)
    return E


def block_energy_row(q, k, N, block_q, block_k, scale, h, qb):
    """One row E[h, qb, :] of ``block_energy`` (for sampled checks at full size)."""
    nkb = -(-N // block_k)
    r0, r1 = qb * block_q, min(qb * block_q + block_q, N)
    if r1 <= r0:
        return np.zeros(nkb)
    qh = np.asarray(q[h, r0:r1], dtype=np.float64)
    kh = np.asarray(k[h, :N], dtype=np.float64)
    return _energy_row(qh, kh, N, block_k, nkb, float(np.float64(scale)))


def topk_count(frac, nkb):
    """k = ceil(frac * nkb), clamped to [1, nkb]."""
    return int(min(nkb, max(1, math.ceil(frac * nkb))))


def _order(row):
    """Key-block indices sorted by (energy descending, index ascending)."""
    row = np.asarray(row, dtype=np.float64)
    idx = np.arange(row.size)
    return np.lexsort((idx, -row))


def select_topk(E, frac):
    """Per row of ``E`` [..., nkb]: 1 for the top-k key blocks, else 0."""
    E = np.asarray(E, dtype=np.float64)
    nkb = E.shape[-1]
    k = topk_count(frac, nkb)
    flat = E.reshape(-1, nkb)
    keep = np.zeros(flat.shape, dtype=np.uint8)
    for r in range(flat.shape[0]):
        keep[r, _order(flat[r])[:k]] = 1
    return keep.reshape(E.shape)


def select_energy(E, eps):
    """Per row: shortest (energy desc, index asc) prefix holding >= (1-eps) of the row's energy."""
    E = np.asarray(E, dtype=np.float64)
    nkb = E.shape[-1]
    flat = E.reshape(-1, nkb)
    keep = np.zeros(flat.shape, dtype=np.uint8)
    for r in range(flat.shape[0]):
        row = flat[r]
        total = 0.0
        for x in row:                       # float64, key-block order
            total += float(x)
        target = (1.0 - float(eps)) * total
        run = 0.0
        for kb in _order(row):
            keep[r, kb] = 1
            run += float(row[kb])           # float64, selection order
            if run >= target:
                break
    return keep.reshape(E.shape)


def min_votes_for(rho, n_inputs):
    """Integer agreement threshold: keep iff votes / I >= rho."""
    v = math.ceil(round(float(rho) * int(n_inputs), 9))
    return int(min(max(v, 0), int(n_inputs)))


def vote(keeps, min_votes, energies=None):
    """Aggregate per-input keep masks.

    ``keeps``: [I, H, nqb, nkb] 0/1; ``energies``: [I, H, nqb, nkb] or None.
    Returns (mask uint8 [H, nqb, nkb], votes int32, energy_sum float32).
    """
    keeps = np.asarray(keeps)
    I = keeps.shape[0]
    votes = keeps.astype(np.int32).sum(axis=0).astype(np.int32)
    esum = np.zeros(keeps.shape[1:], dtype=np.float32)
    if energies is not None:
        energies = np.asarray(energies)
        for n in range(I):                  # float32 running sum, input order
            esum = (esum + energies[n].astype(np.float32)).astype(np.float32)
    mask = (votes >= int(min_votes)).astype(np.uint8)
    H, nqb, nkb = mask.shape
    for h in range(H):
        for qb in range(nqb):
            if mask[h, qb].any():
                continue
            best = None
            for kb in range(nkb):
                key = (int(votes[h, qb, kb]), float(esum[h, qb, kb]), -kb)
                if best is None or key > best[0]:
                    best = (key, kb)
            mask[h, qb, best[1]] = 1
    return mask, votes, esum
