"""Spatial repetition (anchor query rows + broadcast) on the GPU against the oracle (O8).

The row gather is data movement: bit-exact.  Anchor attention is checked on a
small video against the float64 oracle (bf16 bound), equals the plain dense
forward bit for bit when every row is an anchor, and is timed on the Wan
480p shape for Table S4's anchor counts.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

from _util import BF16_MAX_ABS, BF16_MEAN_ABS, assert_close, bf16_pair, to_np64

pytestmark = pytest.mark.gpu


def test_gather_rows_exact():
    rng = np.random.default_rng(1)
    src = torch.from_numpy(rng.standard_normal((3, 2, 50, 64)).astype(np.float32)).cuda().to(torch.bfloat16)
    idx = rng.integers(-3, 50, size=77).astype(np.int32)
    got = cba.gather_rows(src, idx).cpu()
    want = torch.zeros((3, 2, 77, 64), dtype=torch.bfloat16)
    ok = idx >= 0
    want[:, :, torch.from_numpy(np.nonzero(ok)[0])] = src.cpu()[:, :, torch.from_numpy(idx[ok]).long()]
    assert torch.equal(got, want)


@pytest.mark.parametrize("frames,rows,cols,k", [(3, 7, 5, 3), (21, 30, 52, 5), (21, 30, 52, 30), (21, 45, 80, 4),
                                                 (2, 6, 5, 1)])
def test_anchor_plan_matches_the_oracle_mapping(frames, rows, cols, k):
    # calibatt_anchor_plan on the device, bit for bit: gathered query i is the
    # token of its frame's anchor row, every token's output comes from the
    # gathered row of the token on its nearest anchor row, padding is -1.
    N = frames * rows * cols
    Np = (N + 127) // 128 * 128
    plan = cba.anchor_plan(frames, rows, cols, k, Np, "cuda")
    anchors, nearest = oracle.anchor_rows(rows, k)
    per_frame = k * cols
    want_q = np.full(plan.npq, -1, np.int64)
    want_o = np.full(Np, -1, np.int64)
    for f in range(frames):
        for a, ar in enumerate(anchors):
            for c in range(cols):
                want_q[f * per_frame + a * cols + c] = (f * rows + ar) * cols + c
        for r in range(rows):
            slot = anchors.index(nearest[r])
            for c in range(cols):
                want_o[(f * rows + r) * cols + c] = f * per_frame + slot * cols + c
    assert plan.nq == frames * k * cols and plan.npq % 128 == 0 and plan.npq - plan.nq < 128
    assert np.array_equal(plan.idx_q.cpu().numpy(), want_q)
    assert np.array_equal(plan.idx_o.cpu().numpy(), want_o)


@pytest.mark.parametrize("k_anchor", [10, 4, 1])
def test_anchor_attention_small_video(k_anchor):
    frames, rows, cols, H, d = 3, 10, 20, 2, 128
    N = frames * rows * cols
    Np = (N + 127) // 128 * 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 71)
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    plan = cba.anchor_plan(frames, rows, cols, k_anchor, Np, "cuda")
    o = cba.anchor_attention(qd, kd, vd, plan)
    torch.cuda.synchronize()
    want = oracle.anchor_attention(q64, k64, v64, N, frames, rows, cols, k_anchor, cba.default_scale(d))
    mx, mn = assert_close(to_np64(o), want, BF16_MAX_ABS, BF16_MEAN_ABS)
    print(f"PARITY anchor k={k_anchor} of {rows} rows: max_abs={mx:.3e} mean_abs={mn:.3e}")
    if k_anchor == rows:
        bl = cba.compile(torch.ones((H, Np // 128, Np // 128), dtype=torch.uint8, device="cuda"))
        dense = cba.sparse_attn_fwd(qd, kd, vd, bl, N)
        assert torch.equal(o[:, :, :N], dense[:, :, :N])


@pytest.mark.slow
def test_anchor_attention_wan480_timing_and_sampled_parity():
    # Table S4's setting: 30 spatial rows per frame at 480p, attention of k
    # anchor rows against every key, outputs broadcast.
    w = syn.WORKLOADS["wan480_25"]
    g = w.grid
    q, k, v = syn.video_qkv(w)
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    del q, k, v
    scale = cba.default_scale(w.d)
    times = {}
    for k_anchor in (30, 15, 10, 5, 4, 3):
        plan = cba.anchor_plan(g.frames, g.rows, g.cols, k_anchor, w.Np, "cuda")
        bl = cba.compile(torch.ones((w.H, plan.npq // 128, w.Np // 128), dtype=torch.uint8, device="cuda"))
        for _ in range(3):
            o = cba.anchor_attention(qd, kd, vd, plan, bl=bl)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            o = cba.anchor_attention(qd, kd, vd, plan, bl=bl)
        e1.record()
        torch.cuda.synchronize()
        times[k_anchor] = e0.elapsed_time(e1) / 10
        if k_anchor == 5:
            # 16 whole query blocks (2 048 tokens: every row of each block,
            # anchors and their copies), spread over heads and positions
            rng = np.random.default_rng(3)
            picks = [(int(rng.integers(w.H)), int(qb)) for qb in
                     [0, w.nqb - 1] + rng.choice(np.arange(1, w.nqb - 1), 14, replace=False).tolist()]
            errs = []
            for h, qb in picks:
                toks = list(range(qb * 128, min((qb + 1) * 128, w.N)))
                want = oracle.anchor_attention_tokens(q64, k64, v64, w.N, g.frames, g.rows, g.cols, k_anchor, scale,
                                                      0, h, toks)
                errs.append(np.abs(to_np64(o[0, h, toks[0]:toks[-1] + 1]) - want).ravel())
            err = np.concatenate(errs)
            print(f"PARITY anchor wan480 k=5 on {len(picks)} whole query blocks: max_abs={err.max():.3e} "
                  f"mean_abs={err.mean():.3e}")
            assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS
    dense = times[30]
    print("TIMING anchor wan480 (gather + forward + broadcast, ms): " +
          ", ".join(f"k={k} {t:.2f} ({100 * (1 - k / 30):.1f}% rows skipped, {dense / t:.2f}x)" for k, t in times.items()))
