"""GPU compile (calibatt_compile) is bit-exact with the oracle's compile."""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

pytestmark = pytest.mark.gpu


def compare(masks, dedup):
    bl = cba.compile(torch.from_numpy(masks).cuda(), dedup=dedup)
    got = bl.to_numpy()
    want = oracle.compile_blocklist(masks, dedup=(dedup != cba.DEDUP_NONE))
    for key in ("n_pat", "nnz_pat", "nnz"):
        assert got[key] == want[key], key
    for key in ("row_base", "row_pat", "pat_ptr", "pat_off", "csr_row_ptr", "csr_col"):
        assert np.array_equal(got[key], want[key]), key
    return bl


@pytest.mark.parametrize("dedup", [cba.DEDUP_HASH, cba.DEDUP_NONE, cba.DEDUP_HASH_WEAK])
def test_random_masks(dedup):
    rng = np.random.default_rng(1)
    masks = (rng.random((5, 37, 41)) < 0.2).astype(np.uint8)
    masks[2, 5] = 0
    masks[4] = 0
    compare(masks, dedup)


@pytest.mark.parametrize("dedup", [cba.DEDUP_HASH, cba.DEDUP_HASH_WEAK])
def test_structured_masks(dedup):
    masks = syn.structured_block_mask(6, 64, 64, [0.1, 0.2, 0.3, 0.4, 0.5, 0.6], 7, 52, 1560)
    compare(masks, dedup)


def test_banded_and_degenerate():
    n = 300
    band = np.zeros((2, n, n), np.uint8)
    for i in range(n):
        band[0, i, max(0, i - 5):i + 6] = 1
    band[1] = 1
    bl = compare(band, cba.DEDUP_HASH)
    assert bl.n_pat == 5 + 2 + 1          # band patterns + full row; closed form w + 2, plus the all-ones row
    compare(np.zeros((3, 4, 5), np.uint8), cba.DEDUP_HASH)
    compare(np.ones((1, 1, 1), np.uint8), cba.DEDUP_HASH)
    compare(np.ones((2, 3, 700), np.uint8), cba.DEDUP_NONE)


@pytest.mark.slow
def test_sweep_maps_full_size():
    # 4800 (layer, timestep, head) maps of 256 x 256 blocks, densities 0.1 - 0.6
    dens = np.random.default_rng(1000).uniform(0.1, 0.6, 4800)
    masks = np.concatenate([syn.structured_block_mask(1, 256, 256, dens[m], 1000 + m, 52, 1560)
                            for m in range(0, 4800, 4)], axis=0)   # every 4th map: 1200 maps
    bl = cba.compile(torch.from_numpy(masks).cuda())
    got = bl.to_numpy()
    want = oracle.compile_blocklist(masks)
    for key in ("row_base", "row_pat", "pat_ptr", "pat_off", "csr_row_ptr", "csr_col"):
        assert np.array_equal(got[key], want[key]), key


def test_blocklist_kept_counts_match_the_masks():
    # calibatt_blocklist_kept: kept blocks of any map range, from the pattern pool.
    rng = np.random.default_rng(44)
    masks = (rng.random((9, 11, 23)) < rng.random((9, 1, 1))).astype(np.uint8)
    masks[3] = 0
    bl = cba.compile(torch.from_numpy(masks).cuda())
    for mo, n in ((0, 9), (0, 1), (3, 1), (2, 5), (8, 1)):
        assert bl.kept_blocks(mo, n) == int(masks[mo:mo + n].sum())


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs a second visible GPU")
def test_forward_and_energy_on_a_second_device_after_the_first():
    # Launch set-up (shared-memory limits, SM counts) is per device: the same
    # process runs the kernels on device 0, then on device 1.
    from block_sparse_attention_cross_b200 import synthetic as syn
    H, N, Np, d = 2, 1000, 1024, 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 5)
    mask = np.ones((H, 8, 8), np.uint8)
    outs = []
    for dev in (0, 1):
        with torch.cuda.device(dev):
            t = [torch.from_numpy(x).to(f"cuda:{dev}").to(torch.bfloat16) for x in (q, k, v)]
            bl = cba.compile(torch.from_numpy(mask).to(f"cuda:{dev}"))
            outs.append(cba.sparse_attn_fwd(*t, bl, N).cpu())
            E = cba.block_energy(t[0][0], t[1][0], N)
            assert torch.allclose(E[:, :, :].sum(-1), torch.ones_like(E[:, :, 0]), atol=1e-4)
    assert torch.equal(outs[0], outs[1])
