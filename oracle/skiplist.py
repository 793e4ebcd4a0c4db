"""O7 -- the pages' interval skip-list storage of a mask dictionary.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The paper page stores, per layer, a padded 2-D array with one row per
(timestep, head, query block) holding the row's kept/skipped interval pairs
(Figure S10); Figure S9 counts the intervals per row (95% of 720p rows need
at most 50, of a theoretical 295).  Figure S10 trims each layer's width to its
widest row and then merges outlier rows to lower that width; Table S3 lists
the sizes at 100% (no merge), 99% and 95% and a slightly lower sparsity after
merging.  Readings taken, in order:

1. ``interval_counts`` -- a row's intervals are its maximal runs of
   consecutive kept key blocks.
2. ``merge_row`` -- a row with more than ``width`` intervals is merged by
   filling its smallest gaps (runs of skipped blocks between two kept runs;
   ties to the leftmost) until ``width`` intervals remain: the filled blocks
   are computed too, which is the sparsity the merge gives up.
3. ``skiplist_bytes`` -- one interval is a pair of int32 indices (8 bytes);
   a layer of R rows at width W takes R * W * 8 bytes.  Full allocation uses
   the most intervals any row can have, ceil(nkb / 2); trimming uses the
   layer's widest row; merging at x% uses the nearest-rank x-th percentile of
   the layer's interval counts.
"""

from __future__ import annotations

import math

import numpy as np


def interval_counts(masks):
    """[n_maps, nqb] number of maximal runs of kept blocks per row."""
    m = np.asarray(masks) != 0
    starts = m & ~np.concatenate([np.zeros(m.shape[:-1] + (1,), bool), m[..., :-1]], axis=-1)
    return starts.sum(axis=-1)


def _gaps(row):
    """(start, length) of every run of skipped blocks between two kept blocks."""
    kept = [i for i, v in enumerate(row) if v]
    gaps = []
    for a, b in zip(kept, kept[1:]):
        if b > a + 1:
            gaps.append((a + 1, b - a - 1))
    return gaps


def merge_row(row, width):
    """The row with its smallest gaps filled until at most ``width`` intervals remain."""
    row = np.array(row, dtype=np.uint8)
    gaps = _gaps(row)
    excess = len(gaps) + 1 - width if gaps or row.any() else 0
    if excess <= 0:
        return row
    for start, length in sorted(gaps, key=lambda g: (g[1], g[0]))[:excess]:
        row[start:start + length] = 1
    return row


def merge_masks(masks, width_per_map):
    """Every row of map i merged to at most width_per_map[i] intervals."""
    out = np.array(masks, dtype=np.uint8)
    for i in range(out.shape[0]):
        for qb in range(out.shape[1]):
            out[i, qb] = merge_row(out[i, qb], int(width_per_map[i]))
    return out


def nearest_rank(values, pct):
    """Nearest-rank percentile: the smallest value with at least pct% of the values at or below it."""
    v = np.sort(np.asarray(values).ravel())
    k = max(1, math.ceil(pct / 100.0 * v.size))
    return int(v[k - 1])


def skiplist_bytes(counts, maps_per_layer, nkb, pct=100.0):
    """Bytes of the padded per-layer interval arrays; counts [n_maps, nqb]."""
    counts = np.asarray(counts)
    n_layers = counts.shape[0] // maps_per_layer
    full = trimmed = merged = 0
    for l in range(n_layers):
        c = counts[l * maps_per_layer:(l + 1) * maps_per_layer]
        rows = c.size
        full += rows * math.ceil(nkb / 2) * 8
        trimmed += rows * int(c.max()) * 8
        merged += rows * nearest_rank(c, pct) * 8
    return {"full": full, "trimmed": trimmed, "merged": merged}
