"""O6 -- timestep sharing of calibrated masks.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The paper page describes masks calibrated per (layer, head, timestep) and
notes that masks of consecutive late denoising steps are alike (Figure S11:
the intersection-over-union of the skipped-block masks of two timesteps,
averaged over layers and heads), and that timestep sharing "clusters masks
with pair-wise IoU >= tau" (Table S3) to shrink the stored dictionary.  The
pages leave the rest open; the readings taken here, in order:

1. ``skipped_iou`` -- for two masks of one (layer, head), the IoU of their
   *skipped* block sets: |S1 & S2| / |S1 | S2| with S = {blocks with mask 0};
   two masks that skip nothing are identical (IoU 1).
2. ``timestep_clusters`` -- per layer, the similarity of timesteps t1, t2 is
   the mean over heads of their skipped-block IoU (as in Figure S11).
   Timesteps are grouped into runs of *consecutive* steps (Figure S11:
   sharing across consecutive steps) greedily in timestep order: step t joins
   the current run when its similarity with every member of the run is at
   least tau ("pair-wise"), otherwise it starts a new run.
3. ``share_masks`` -- a run stores one mask per head: the union of its
   members' kept blocks, so no block that any member keeps is skipped.

Layout: masks [L, T, H, nqb, nkb] (the dictionary order map = (l T + t) H + h);
shared masks [C, H, nqb, nkb] with the runs numbered in (layer, time) order.
"""

from __future__ import annotations

import numpy as np


def skipped_iou(m1, m2):
    """IoU of the skipped-block sets of two masks (any shape, nonzero = kept)."""
    s1 = np.asarray(m1) == 0
    s2 = np.asarray(m2) == 0
    union = int(np.count_nonzero(s1 | s2))
    if union == 0:
        return 1.0
    return int(np.count_nonzero(s1 & s2)) / union


def timestep_similarity(masks):
    """[L, T, T] float64: mean over heads of the skipped-block IoU."""
    L, T, H = masks.shape[:3]
    sim = np.ones((L, T, T))
    for l in range(L):
        for t1 in range(T):
            for t2 in range(T):
                if t1 != t2:
                    sim[l, t1, t2] = np.mean([skipped_iou(masks[l, t1, h], masks[l, t2, h]) for h in range(H)])
    return sim


def timestep_clusters(masks, tau):
    """[L, T] int32 run index of every timestep (runs numbered from 0 in each layer)."""
    sim = timestep_similarity(masks)
    L, T = masks.shape[:2]
    out = np.zeros((L, T), np.int32)
    for l in range(L):
        run = [0]
        cid = 0
        for t in range(1, T):
            if all(sim[l, t, s] >= tau for s in run):
                run.append(t)
            else:
                cid += 1
                run = [t]
            out[l, t] = cid
    return out


def share_masks(masks, clusters):
    """Union masks [C, H, nqb, nkb] uint8 and the map offset (C-index * H) of every (l, t)."""
    L, T, H = masks.shape[:3]
    shared = []
    offset = np.zeros((L, T), np.int64)
    for l in range(L):
        for c in range(int(clusters[l].max()) + 1):
            members = [t for t in range(T) if clusters[l, t] == c]
            u = np.zeros((H,) + masks.shape[3:], bool)
            for t in members:
                u |= masks[l, t] != 0
            for t in members:
                offset[l, t] = len(shared) * H
            shared.append(u.astype(np.uint8))
    return np.stack(shared), offset
