"""Seeded input generators: shapes, exact densities, structure, bf16 rounding,
and the geometry the CalibAtt paper page prints (tests/golden/geometry.json)."""

import json
from pathlib import Path

import numpy as np
import torch

from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

GOLDEN = Path(__file__).resolve().parent / "golden"


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 10
    x[:4] = [1.00390625, 1.01171875, -3.0e38, 0.0]  # halfway cases and extremes
    ours = syn.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = syn.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_geometry_matches_pages():
    g = json.loads((GOLDEN / "geometry.json").read_text())
    assert syn.WORKLOADS["wan480_25"].N == g["wan480_sequence_length"]["value"]
    assert syn.WORKLOADS["wan720_20"].N == g["wan720_sequence_length"]["value"]
    wan = syn.WORKLOADS["wan480_25"].grid
    assert 2 * wan.rows * wan.cols == g["wan480_two_frames_tokens"]["value"]
    for k, sps in zip(g["table_s4_anchor_rows"]["k"], g["table_s4_anchor_rows"]["sparsity_pct"]):
        assert round(100 * (1 - k / wan.rows), 1) == sps
    w720 = syn.WORKLOADS["wan720_20"]
    assert (w720.Np // w720.block) // 2 == g["wan720_max_intervals_per_row"]["value"]


def test_random_block_mask_exact():
    w = syn.WORKLOADS["tiny_fp32"]
    m = syn.workload_mask(w)
    assert m.shape == (2, 16, 16)
    for h in range(2):
        assert m[h].sum() == 128
        assert np.all(np.diag(m[h]) == 1)
    assert np.array_equal(m, syn.workload_mask(w))


def test_structured_masks_exact_density_and_dedup_gain():
    for name in ("wan480_25", "wan720_20", "mochi_20"):
        w = syn.WORKLOADS[name]
        m = syn.workload_mask(w, n_maps=2)
        nkb = w.Np // w.block
        assert m.sum(axis=(1, 2)).tolist() == [round(w.density * w.nqb * nkb)] * 2
        for h in range(2):
            assert np.all(np.diag(m[h]) == 1)
        if w.grid.text_tokens:
            first_text = w.grid.video_tokens // w.block
            assert np.all(m[:, :, first_text:] == 1)
        else:
            bl = oracle.compile_blocklist(m)
            assert bl["nnz_pat"] < bl["nnz"]          # repetition is there to be found
    m = syn.structured_block_mask(3, 256, 256, [0.1, 0.35, 0.6], 1000, 52, 1560)
    assert m.sum(axis=(1, 2)).tolist() == [round(d * 65536) for d in (0.1, 0.35, 0.6)]


def test_video_qkv_shapes_and_padding():
    w = syn.Workload("t", 1, 2, syn.VideoGrid(2, 3, 50), 64, "bf16", 128, 0.25,
                     {"base": 1, "noise_q": 2, "noise_k": 3, "v": 4})
    q, k, v = syn.video_qkv(w)
    assert q.shape == (1, 2, 384, 64) and w.N == 300
    assert np.all(q[:, :, 300:] == 0) and np.all(v[:, :, 300:] == 0)
    q2, k2, v2 = syn.video_qkv(w)
    assert np.array_equal(q, q2) and np.array_equal(v, v2)
    qa, ka = syn.video_qkv(w, with_v=False, input_index=0)
    qb, kb = syn.video_qkv(w, with_v=False, input_index=1)
    assert not np.array_equal(qa, qb)
    # shared structure: Q and K of the same token are strongly correlated
    c = np.corrcoef(q[0, 0, :300].ravel(), k[0, 0, :300].ravel())[0, 1]
    assert c > 0.9


def test_anchor_rows_through_the_c_abi_match_the_oracle():
    # calibatt_anchor_rows is host arithmetic in the library (no device work):
    # anchors and nearest-anchor mapping equal the oracle's for every k of the
    # pages' 30-row frames and for odd small frames; sizes of the gathered
    # query tensor follow the geometry.
    import ctypes
    import oracle
    import block_sparse_attention_cross_b200 as cba
    for rows in (30, 45, 7, 1):
        for k in range(1, rows + 1):
            assert cba.anchor_rows(rows, k) == oracle.anchor_rows(rows, k)
    lib = cba.load()
    nq, npq = ctypes.c_int(0), ctypes.c_int(0)
    assert lib.calibatt_anchor_plan_size(21, 30, 52, 5, ctypes.byref(nq), ctypes.byref(npq)) == 0
    assert (nq.value, npq.value) == (21 * 5 * 52, 5504)
    assert lib.calibatt_anchor_plan_size(2, 30, 52, 31, ctypes.byref(nq), ctypes.byref(npq)) == cba._lib.E_INVALID
