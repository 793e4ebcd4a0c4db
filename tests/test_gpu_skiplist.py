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


@pytest.mark.parametrize("maps_per_layer,pcts", [(3, (100.0, 99.0, 95.0, 50.0)), (12, (95.0, 12.5)), (1, (100.0,))])
def test_skiplist_sizes_match_the_oracle(maps_per_layer, pcts):
    # calibatt_skiplist_sizes: per-layer maximum and nearest-rank percentile
    # widths of the interval counts and the byte totals, bit for bit against
    # the oracle; the per-map widths drive the merge to the oracle's masks.
    rng = np.random.default_rng(9)
    n_maps, nqb, nkb = 12, 9, 75
    dens = rng.choice([0.05, 0.2, 0.5, 0.9], size=(n_maps, nqb, 1))
    masks = (rng.random((n_maps, nqb, nkb)) < dens).astype(np.uint8)
    md = torch.from_numpy(masks).cuda()
    rep = cba.skiplist_report(md, maps_per_layer, pcts)
    counts = oracle.interval_counts(masks)
    layers = n_maps // maps_per_layer
    per_layer = counts.reshape(layers, -1)
    assert rep["layer_max"] == per_layer.max(axis=1).tolist()
    assert rep["intervals_max"] == int(counts.max()) and rep["intervals_p95"] == oracle.nearest_rank(counts, 95.0)
    for m, pct in zip(rep["merged"], pcts):
        want = oracle.skiplist_bytes(counts, maps_per_layer, nkb, pct=pct)
        assert (rep["skiplist_full_bytes"], rep["skiplist_trimmed_bytes"], m["bytes"]) == \
            (want["full"], want["trimmed"], want["merged"])
        widths = [oracle.nearest_rank(per_layer[l], pct) for l in range(layers)]
        assert m["layer_width"] == widths
        merged = oracle.merge_masks(masks, np.repeat(widths, maps_per_layer))
        assert m["filled_blocks"] == int(merged.sum()) - int(masks.sum())
    bl = oracle.compile_blocklist(masks)
    assert rep["csr_bytes"] == (n_maps * nqb + 1) * 8 + int(masks.sum()) * 2
    assert rep["pattern_pool_bytes"] == n_maps * nqb * 8 + bl["pat_ptr"].size * 4 + bl["pat_off"].size * 2


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
