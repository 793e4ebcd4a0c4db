"""Spatial-similarity score and repetition dictionary on the GPU against the oracle (O9).

The score is floating point: compared with the float64 oracle within 1e-4.
The dictionary's flags are a floating-point decision: on the GPU's own
per-input scores the oracle's mean-and-threshold (float32, input order) must
give the same flags bit for bit; against the float64 scores, flags may
differ only where the mean is within 1e-4 of tau.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

from _util import bf16_pair

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _inputs(grid, H, d, row_scale, n=0, seed=60):
    w = syn.Workload("sim", 1, H, grid, d, "bf16", 128, 0.25, {"base": seed, "noise_q": seed + 1,
                                                              "noise_k": seed + 2, "v": seed + 3})
    q, k = syn.video_qkv(w, with_v=False, input_index=n, row_scale=row_scale)
    return w, bf16_pair(q[0]), bf16_pair(k[0])


@pytest.mark.parametrize("d,grid", [(128, syn.VideoGrid(3, 6, 10)), (64, syn.VideoGrid(2, 7, 23, text_tokens=19)),
                                    (128, syn.VideoGrid(2, 30, 52))])
def test_spatial_similarity_small(d, grid):
    H = 4
    w, (q64, qd), (k64, kd) = _inputs(grid, H, d, [1.0, 0.0, 0.3, 0.05])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = cba.spatial_similarity(qd, kd, w.N, grid.frames, grid.rows, grid.cols, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    want = oracle.spatial_similarity(q64, k64, w.N, grid.frames, grid.rows, grid.cols, cba.default_scale(d))
    err = np.abs(got.cpu().numpy().astype(np.float64) - want)
    print(f"PARITY spatial similarity d={d} grid={grid.frames}x{grid.rows}x{grid.cols}+{grid.text_tokens}: "
          f"scores {np.round(want, 4).tolist()} max_abs={err.max():.2e}")
    assert err.max() <= TOL
    # deterministic: a second call gives the same bits
    assert torch.equal(got, cba.spatial_similarity(qd, kd, w.N, grid.frames, grid.rows, grid.cols))


def test_repetition_dictionary_flags():
    # 3 calibration inputs of 8 heads with different row structure; tau put
    # between the heads' scores so that some are flagged and some are not.
    grid, H, d = syn.VideoGrid(3, 8, 16), 8, 128
    rs = [1.0, 0.0, 0.5, 0.02, 0.8, 0.1, 0.0, 0.3]
    scores_g, scores_o = [], []
    for n in range(3):
        w, (q64, qd), (k64, kd) = _inputs(grid, H, d, rs, n=n)
        scores_g.append(cba.spatial_similarity(qd, kd, w.N, grid.frames, grid.rows, grid.cols))
        scores_o.append(oracle.spatial_similarity(q64, k64, w.N, grid.frames, grid.rows, grid.cols,
                                                  cba.default_scale(d)))
    sg = torch.stack(scores_g)
    so = np.stack(scores_o)
    tau = float(np.median(so.mean(axis=0)))
    mean, flags = cba.repetition_flags(sg, tau)
    m_o, f_o = oracle.repetition_flags(sg.cpu().numpy(), tau)
    assert np.array_equal(mean.cpu().numpy(), m_o) and np.array_equal(flags.cpu().numpy(), f_o)
    f64 = (so.mean(axis=0) >= tau).astype(np.uint8)
    near = np.abs(so.mean(axis=0) - tau) < TOL
    assert not ((flags.cpu().numpy() != f64) & ~near).any()
    assert 0 < int(flags.sum()) < H
    print(f"PARITY repetition dictionary: tau={tau:.4f} flags {flags.cpu().tolist()} (bit-exact on GPU scores)")


@pytest.mark.slow
def test_spatial_similarity_wan480_and_flags():
    # The Wan 480p shape (40 heads, 32 760 tokens) with a per-head spatial-row
    # weight; the oracle checks 3 heads; the dictionary flags heads at the
    # pages' tau = 0.87.
    w = syn.WORKLOADS["wan480_25"]
    g = w.grid
    rs = np.linspace(0.0, 1.0, w.H)
    scores = []
    for n in range(2):
        q, k = syn.video_qkv(w, with_v=False, input_index=n, row_scale=rs)
        q64, qd = bf16_pair(q[0])
        k64, kd = bf16_pair(k[0])
        del q, k
        s = cba.spatial_similarity(qd, kd, w.N, g.frames, g.rows, g.cols)
        scores.append(s)
        if n == 0:
            heads = [0, 20, 39]
            want = oracle.spatial_similarity(q64[heads], k64[heads], w.N, g.frames, g.rows, g.cols,
                                             cba.default_scale(w.d))
            err = np.abs(s.cpu().numpy()[heads].astype(np.float64) - want)
            print(f"PARITY spatial similarity wan480 heads {heads}: {np.round(want, 4).tolist()} "
                  f"max_abs={err.max():.2e}")
            assert err.max() <= TOL
        del q64, k64, qd, kd
    mean, flags = cba.repetition_flags(torch.stack(scores), 0.87)
    m_o, f_o = oracle.repetition_flags(torch.stack(scores).cpu().numpy(), 0.87)
    assert np.array_equal(flags.cpu().numpy(), f_o)
    print(f"PARITY repetition dictionary wan480 tau=0.87: {int(flags.sum())} of {w.H} heads flagged; "
          f"mean scores {np.round(mean.cpu().numpy()[[0, 10, 20, 30, 39]], 3).tolist()} (heads 0,10,20,30,39)")
