"""Interval skip-list view of mask dictionaries on the GPU against the oracle (O7).

Interval counts and merged masks are integer work: bit-exact.  The storage
report of the 4 800-map sweep dictionary (480p) and of the 720p dictionary is
printed: the pages' padded interval arrays (full, trimmed, merged at 99% and
95%) next to this library's CSR and pattern pool.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

pytestmark = pytest.mark.gpu


def test_counts_and_merge_match_oracle():
    rng = np.random.default_rng(12)
    n_maps, nqb, nkb = 6, 7, 45
    dens = rng.choice([0.05, 0.3, 0.6, 0.95], size=(n_maps, 1, 1))
    masks = (rng.random((n_maps, nqb, nkb)) < dens).astype(np.uint8)
    masks[0, 3] = 0                                   # an empty row
    masks[1, 2] = 1                                   # a full row
    md = torch.from_numpy(masks).cuda()
    assert np.array_equal(cba.interval_counts(md).cpu().numpy(), oracle.interval_counts(masks))
    width = rng.integers(1, 6, size=n_maps).astype(np.int32)
    filled = cba.merge_intervals(md, width)
    want = oracle.merge_masks(masks, width)
    assert np.array_equal(md.cpu().numpy(), want)
    assert filled == int(want.sum()) - int(masks.sum())
    assert (oracle.interval_counts(want) <= np.maximum(width, 1)[:, None]).all()


def _report(masks_np, maps_per_layer, name):
    md = torch.from_numpy(masks_np).cuda()
    assert np.array_equal(cba.interval_counts(md).cpu().numpy(), oracle.interval_counts(masks_np))
    rep = cba.skiplist_report(md, maps_per_layer)
    want = oracle.skiplist_bytes(oracle.interval_counts(masks_np), maps_per_layer, masks_np.shape[2], pct=95.0)
    assert rep["skiplist_full_bytes"] == want["full"] and rep["skiplist_trimmed_bytes"] == want["trimmed"]
    assert rep["merged"][-1]["bytes"] == want["merged"]
    mb = lambda b: f"{b / 2**20:.1f} MiB"
    merged = ", ".join(f"{m['pct']:.0f}% {mb(m['bytes'])} (density {m['density']:.4f})" for m in rep["merged"])
    print(f"STORAGE {name}: {rep['rows']} rows, density {rep['density']:.4f}, intervals max {rep['intervals_max']} "
          f"p95 {rep['intervals_p95']}; skip lists full {mb(rep['skiplist_full_bytes'])}, trimmed "
          f"{mb(rep['skiplist_trimmed_bytes'])}, merged {merged}; CSR {mb(rep['csr_bytes'])}, "
          f"pattern pool {mb(rep['pattern_pool_bytes'])}")
    return rep


@pytest.mark.slow
def test_sweep_dictionary_storage_and_merge_subset():
    w = syn.WORKLOADS["wan480_25"]
    masks = syn.sweep_masks(w, 40, 3)                      # 4 800 maps; a layer = 3 timesteps x 40 heads
    _report(masks, 3 * w.H, "sweep 480p 40x3x40")
    sub = masks[:80].copy()                                 # merge parity on 80 maps (20 480 rows)
    counts = oracle.interval_counts(sub)
    width = np.array([oracle.nearest_rank(counts[i], 90.0) for i in range(80)], np.int32)
    md = torch.from_numpy(sub).cuda()
    cba.merge_intervals(md, width)
    assert np.array_equal(md.cpu().numpy(), oracle.merge_masks(sub, width))


@pytest.mark.slow
def test_wan720_dictionary_storage():
    w = syn.WORKLOADS["wan720_20"]
    masks = syn.workload_mask(w)                            # 40 heads x 591 x 591
    _report(masks, w.H, "wan720 20% 40 heads")
    sub = masks[:3].copy()
    width = np.array([8, 3, 20], np.int32)
    md = torch.from_numpy(sub).cuda()
    cba.merge_intervals(md, width)
    assert np.array_equal(md.cpu().numpy(), oracle.merge_masks(sub, width))
