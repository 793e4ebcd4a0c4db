"""Timestep sharing of calibrated masks on the GPU against the oracle (O6).

Runs are decided from exact integer pair counts, so the run of every
(layer, timestep), the shared union masks and the map offsets must match the
oracle exactly.  The shared dictionary then drives the forward kernel.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

from _util import BF16_MAX_ABS, BF16_MEAN_ABS, assert_lse, bf16_pair, to_np64

pytestmark = pytest.mark.gpu


def drifting_masks(L, T, H, nb, seed):
    # masks whose kept blocks flip from step to step at a per-layer rate
    # (1% ... 40%), so the layers split into runs of very different lengths
    rng = np.random.default_rng(seed)
    base = rng.random((L, 1, H, nb, nb)) < 0.4
    rates = np.array([0.01, 0.05, 0.15, 0.4])[:L].reshape(L, 1, 1, 1, 1)
    flips = rng.random((L, T, H, nb, nb)) < rates
    return (base ^ (np.cumsum(flips, axis=1) % 2).astype(bool)).astype(np.uint8)


def global_runs(cl):
    out = np.zeros_like(cl)
    base = 0
    for l in range(cl.shape[0]):
        out[l] = cl[l] + base
        base += int(cl[l].max()) + 1
    return out, base


@pytest.mark.parametrize("tau", [0.3137, 0.6071, 0.8923])
def test_clusters_and_union_match_oracle(tau):
    L, T, H, nb = 4, 9, 3, 24
    masks = drifting_masks(L, T, H, nb, 5)
    run_of, n_runs = cba.timestep_clusters(torch.from_numpy(masks).cuda(), tau)
    want, n_want = global_runs(oracle.timestep_clusters(masks, tau))
    assert n_runs == n_want
    assert np.array_equal(run_of.numpy(), want)
    shared, offset = cba.share_timesteps(torch.from_numpy(masks).cuda(), tau)
    s_want, o_want = oracle.share_masks(masks, oracle.timestep_clusters(masks, tau))
    assert np.array_equal(shared.cpu().numpy(), s_want.reshape(-1, nb, nb))
    assert np.array_equal(offset.numpy(), o_want)
    print(f"PARITY share tau={tau}: {n_runs} runs of {L * T} (layer, timestep) masks, runs and unions exact")


@pytest.mark.slow
def test_sweep_dictionary_sharing_drives_forward():
    # The 40 x 3 x 40 sweep dictionary of the Wan 480p shape with its masks
    # made to drift slowly over the 3 timesteps, shared at tau = 0.55, then
    # compiled and used by the forward kernel on sampled query blocks.
    w = syn.WORKLOADS["wan480_25"]
    masks = syn.sweep_masks(w, 40, 3).reshape(40, 3, w.H, w.nqb, w.nqb)
    rng = np.random.default_rng(9)
    masks[:, 1] = masks[:, 0] ^ (rng.random(masks[:, 1].shape) < 0.02)
    masks[:, 1] = np.maximum(masks[:, 1], np.eye(w.nqb, dtype=np.uint8))
    tau = 0.55
    shared, offset = cba.share_timesteps(torch.from_numpy(masks).cuda(), tau)
    s_want, o_want = oracle.share_masks(masks, oracle.timestep_clusters(masks, tau))
    assert np.array_equal(shared.cpu().numpy(), s_want.reshape(-1, w.nqb, w.nqb))
    assert np.array_equal(offset.numpy(), o_want)
    bl = cba.compile(shared)
    q, k, v = syn.video_qkv(w)
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    scale = cba.default_scale(w.d)
    for layer, t in ((0, 1), (21, 0)):
        mo = int(offset[layer, t])
        o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, w.N, scale=scale, map_offset=mo, return_lse=True)
        torch.cuda.synchronize()
        sm = s_want.reshape(-1, w.nqb, w.nqb)[mo:mo + w.H]
        errs = []
        for h, qb in [(0, 0), (w.H - 1, w.nqb - 1), (7, 101), (23, 200)]:
            O, L = oracle.masked_attention_rows(q64, k64, v64, sm, w.N, 128, 128, scale, 0, h, qb)
            rows = slice(qb * 128, (qb + 1) * 128)
            errs.append(np.abs(to_np64(o[0, h, rows]) - O).ravel())
            assert_lse(lse[0, h, rows].cpu().numpy(), L, 1e-3)
        err = np.concatenate(errs)
        assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS
    runs = int(shared.shape[0] // w.H)
    print(f"PARITY share sweep tau={tau}: {runs} runs of 120 calls; forward on shared masks max_abs={err.max():.3e}")
