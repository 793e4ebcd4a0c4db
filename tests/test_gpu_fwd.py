"""GPU parity of calibatt_sparse_attn_fwd against the float64 oracle.

bf16 (tcgen05 tensor-core kernel): O within max-abs 2e-2 and mean-abs 2e-3,
LSE within 1e-3.  fp32 (FFMA kernel): O within 1e-5, LSE within 1e-5.
Small cases are compared on every row; full-size workloads on sampled query
blocks that the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

from _util import (BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, assert_close, assert_lse, bf16_pair, fp32_pair,
                   to_np64)

pytestmark = pytest.mark.gpu


def run_full_compare(q, k, v, mask, N, block, dtype, d, B=1, H=None, map_offset=0, lse_tol=None):
    """Whole-tensor parity of one small case."""
    pair = bf16_pair if dtype == "bf16" else fp32_pair
    q64, qd = pair(q)
    k64, kd = pair(k)
    v64, vd = pair(v)
    bl = cba.compile(torch.from_numpy(mask).cuda(), block_q=block, block_k=block)
    H = q.shape[1]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = cba.default_scale(d)
    o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, N, scale=scale, map_offset=map_offset, return_lse=True,
                                 status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    O, L = oracle.masked_attention(q64, k64, v64, mask[map_offset:map_offset + H], N, block, block, scale)
    if dtype == "bf16":
        mx, mn = assert_close(to_np64(o), O, BF16_MAX_ABS, BF16_MEAN_ABS)
        assert_lse(lse.cpu().numpy(), L, lse_tol or 1e-3)
    else:
        mx, mn = assert_close(to_np64(o), O, FP32_MAX_ABS)
        assert_lse(lse.cpu().numpy(), L, lse_tol or 1e-5)
    print(f"PARITY {dtype} N={N} d={d} block={block} max_abs={mx:.3e} mean_abs={mn:.3e}")
    return mx, mn


def test_fp32_tiny_config():
    w = syn.WORKLOADS["tiny_fp32"]
    q, k, v = syn.normal_qkv(w.B, w.H, w.N, w.Np, w.d, w.seeds["data"])
    mask = syn.workload_mask(w)
    run_full_compare(q, k, v, mask, w.N, w.block, "fp32", w.d)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 128), (128, 64)])
def test_fp32_ragged_with_empty_rows(d, block):
    N, Np, H = 1000, 1024, 2
    q, k, v = syn.normal_qkv(2, H, N, Np, d, 7)
    nb = Np // block
    mask = (np.random.default_rng(3).random((H + 1, nb, nb)) < 0.4).astype(np.uint8)
    mask[0, 2, :] = 0                   # empty row
    mask[1, nb - 1, :] = 0              # empty last (padded) row
    mask[1, 0, nb - 1] = 1              # padded key block kept
    run_full_compare(q, k, v, mask, N, block, "fp32", d, map_offset=0)
    run_full_compare(q, k, v, mask, N, block, "fp32", d, map_offset=1)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_small_random_masks(d):
    N, Np, H = 1000, 1024, 3
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 11)
    mask = (np.random.default_rng(5).random((H, 8, 8)) < 0.5).astype(np.uint8)
    mask[0, 3, :] = 0                   # empty row
    mask[1, :, 7] = 1                   # padded key block everywhere
    mask[2, 7, :] = 1                   # padded query block sees all
    run_full_compare(q, k, v, mask, N, 128, "bf16", d)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_full_mask_is_dense(d):
    N, Np, H = 2040, 2048, 2
    q, k, v = syn.normal_qkv(2, H, N, Np, d, 12)
    mask = np.ones((H, 16, 16), np.uint8)
    run_full_compare(q, k, v, mask, N, 128, "bf16", d)


def test_bf16_structured_scores():
    # Wan-like structured Q/K (logit std ~3) with a structured mask, 4 frames
    w = syn.Workload("wan_small", 2, 2, syn.VideoGrid(4, 30, 52), 128, "bf16", 128, 0.3,
                     {"base": 10, "noise_q": 11, "noise_k": 12, "v": 13, "mask": 14})
    q, k, v = syn.video_qkv(w)
    mask = syn.workload_mask(w)
    run_full_compare(q, k, v, mask, w.N, 128, "bf16", 128)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_large_score_jumps(d):
    # Every query shares a direction u and every key carries u with a
    # magnitude set per 64-key half block (32 levels in random order), so the
    # running row maximum jumps by far more than the kernel's rescale
    # threshold in first and second halves of blocks alike (a float64 walk of
    # these inputs in the kernel's block order counts 11 / 22 such jumps at
    # d = 128, 21 / 27 at d = 64): the redo and O-rescale paths run.
    N, Np, H = 2000, 2048, 2
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 41)
    rng = np.random.default_rng(42)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = (q + 8.0 * u).astype(np.float32)
    g = 12.0 * np.repeat(rng.permutation(32), 64)
    k = (k + g[None, None, :, None] * u).astype(np.float32)
    mask = (rng.random((H, 16, 16)) < 0.5).astype(np.uint8)
    mask[0, 5, :] = 1
    mask[1, :, 15] = 1
    run_full_compare(q, k, v, mask, N, 128, "bf16", d)


def test_bf16_deterministic():
    N, Np, H = 1024, 1024, 2
    q, k, v = syn.normal_qkv(1, H, N, Np, 128, 21)
    _, qd = bf16_pair(q)
    _, kd = bf16_pair(k)
    _, vd = bf16_pair(v)
    mask = (np.random.default_rng(9).random((H, 8, 8)) < 0.5).astype(np.uint8)
    bl = cba.compile(torch.from_numpy(mask).cuda())
    o1, l1 = cba.sparse_attn_fwd(qd, kd, vd, bl, N, return_lse=True)
    o2, l2 = cba.sparse_attn_fwd(qd, kd, vd, bl, N, return_lse=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("dtype,d,hpc", [("bf16", 128, 2), ("bf16", 64, 5), ("fp32", 64, 3)])
def test_streamed_host_buffers_match_device_call(dtype, d, hpc):
    # Same kernel per chunk of heads: the host-buffer call must reproduce the
    # device call bit for bit, O and LSE, with a ragged last chunk and B = 2.
    B, H, N, Np = 2, 5, 2000, 2048
    q, k, v = syn.normal_qkv(B, H, N, Np, d, 51)
    pair = bf16_pair if dtype == "bf16" else fp32_pair
    _, qd = pair(q)
    _, kd = pair(k)
    _, vd = pair(v)
    mask = (np.random.default_rng(6).random((H + 2, 16, 16)) < 0.4).astype(np.uint8)
    mask[1, 3, :] = 0
    bl = cba.compile(torch.from_numpy(mask).cuda())
    o_ref, lse_ref = cba.sparse_attn_fwd(qd, kd, vd, bl, N, map_offset=1, return_lse=True)
    qh, kh, vh = (t.cpu().pin_memory() for t in (qd, kd, vd))
    staging = (torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd),
               torch.empty((B, H, Np), dtype=torch.float32, device="cuda"))
    lse_h = torch.empty((B, H, Np), dtype=torch.float32).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_h = cba.sparse_attn_fwd_streamed(qh, kh, vh, bl, N, staging, map_offset=1, heads_per_chunk=hpc, lse=lse_h,
                                       status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(o_h, o_ref.cpu())
    assert torch.equal(lse_h, lse_ref.cpu())


def sampled_parity(w, mask, qkv=None, n_samples=24, seed=0, map_offset=0):
    """Full-size run; oracle on sampled (head, query block) pairs incl. the first and last block."""
    q, k, v = qkv if qkv is not None else syn.video_qkv(w)
    q64, qd = bf16_pair(q)
    del q
    k64, kd = bf16_pair(k)
    del k
    v64, vd = bf16_pair(v)
    del v
    bl = cba.compile(torch.from_numpy(mask).cuda())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = cba.default_scale(w.d)
    o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, w.N, scale=scale, map_offset=map_offset, return_lse=True,
                                 status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    rng = np.random.default_rng(seed)
    picks = [(0, 0), (w.H - 1, w.nqb - 1)] + [(int(rng.integers(w.H)), int(rng.integers(w.nqb)))
                                              for _ in range(n_samples - 2)]
    errs = []
    for h, qb in picks:
        O, L = oracle.masked_attention_rows(q64, k64, v64, mask[map_offset:], w.N, w.block, w.block, scale, 0, h, qb)
        rows = slice(qb * w.block, (qb + 1) * w.block)
        got = to_np64(o[0, h, rows])
        errs.append(np.abs(got - O))
        assert_lse(lse[0, h, rows].cpu().numpy(), L, 1e-3)
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
    print(f"PARITY {w.name} sampled {len(picks)} query blocks max_abs={err.max():.3e} mean_abs={err.mean():.3e}")
    return err.max(), err.mean()


@pytest.mark.slow
def test_bf16_wan480_full_size_sampled():
    w = syn.WORKLOADS["wan480_25"]
    sampled_parity(w, syn.workload_mask(w))


@pytest.mark.slow
def test_bf16_wan720_full_size_sampled():
    w = syn.WORKLOADS["wan720_20"]
    sampled_parity(w, syn.workload_mask(w), n_samples=12)


@pytest.mark.slow
def test_bf16_mochi_full_size_sampled():
    w = syn.WORKLOADS["mochi_20"]
    sampled_parity(w, syn.workload_mask(w), n_samples=12)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_persistent_schedule_ragged_lists(d):
    # Many work tiles per CTA slot, lists from 0 to all 64 blocks, empty rows
    # interleaved, a batch of 2 and a ragged sequence tail.
    B, H, N, Np = 2, 5, 8000, 8064
    nb = Np // 128
    q, k, v = syn.normal_qkv(B, H, N, Np, d, 31)
    rng = np.random.default_rng(8)
    mask = np.zeros((H, nb, nb), np.uint8)
    for h in range(H):
        for qb in range(nb):
            cnt = int(rng.choice([0, 1, 2, 5, 17, 40, nb]))
            if cnt:
                mask[h, qb, rng.choice(nb, size=cnt, replace=False)] = 1
    run_full_compare(q, k, v, mask, N, 128, "bf16", d)


@pytest.mark.slow
def test_bf16_sweep_dictionary_calls_sampled():
    # 40 layers x 3 timesteps x 40 heads of the Wan 480p shape, each map with
    # its own density in [0.1, 0.6]; a call uses the 40 maps of one
    # (layer, timestep) through map_offset.  Eight seeded calls are checked,
    # every head of each on a sampled query block (the first and the last
    # query block on the first call).
    w = syn.WORKLOADS["wan480_25"]
    masks = syn.sweep_masks(w, 40, 3)
    q, k, v = syn.video_qkv(w)
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    del q, k, v
    bl = cba.compile(torch.from_numpy(masks).cuda())
    assert bl.nnz == int(masks.sum())
    scale = cba.default_scale(w.d)
    rng = np.random.default_rng(4)
    calls = [(0, 0), (39, 2)] + [(int(rng.integers(40)), int(rng.integers(3))) for _ in range(6)]
    for ci, (layer, t) in enumerate(calls):
        mo = (layer * 3 + t) * w.H
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, w.N, scale=scale, map_offset=mo, return_lse=True, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        picks = [(h, int(rng.integers(w.nqb))) for h in range(w.H)]
        if ci == 0:
            picks += [(0, 0), (w.H - 1, w.nqb - 1)]
        errs = []
        for h, qb in picks:
            O, L = oracle.masked_attention_rows(q64, k64, v64, masks[mo:mo + w.H], w.N, 128, 128, scale, 0, h, qb)
            rows = slice(qb * 128, (qb + 1) * 128)
            errs.append(np.abs(to_np64(o[0, h, rows]) - O).ravel())
            assert_lse(lse[0, h, rows].cpu().numpy(), L, 1e-3)
        err = np.concatenate(errs)
        assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (layer, t, err.max(), err.mean())
        print(f"PARITY sweep layer={layer} t={t} heads={w.H} max_abs={err.max():.3e} mean_abs={err.mean():.3e}")


def run_k64_compare(q, k, v, mask, N, d):
    """Whole-tensor parity with 128-row query blocks and 64-key blocks."""
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    bl = cba.compile(torch.from_numpy(mask).cuda(), block_q=128, block_k=64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = cba.default_scale(d)
    o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, N, scale=scale, return_lse=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    O, L = oracle.masked_attention(q64, k64, v64, mask, N, 128, 64, scale)
    mx, mn = assert_close(to_np64(o), O, BF16_MAX_ABS, BF16_MEAN_ABS)
    assert_lse(lse.cpu().numpy(), L, 1e-3)
    print(f"PARITY bf16 128x64 blocks N={N} d={d} max_abs={mx:.3e} mean_abs={mn:.3e}")


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_key_blocks_of_64(d):
    # 128-row query blocks with 64-key blocks: random masks with an empty row,
    # a full row and the padded last key block kept everywhere, ragged N.
    N, Np, H = 2000, 2048, 3
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 61)
    rng = np.random.default_rng(62)
    mask = (rng.random((H, 16, 32)) < 0.4).astype(np.uint8)
    mask[0, 4, :] = 0
    mask[1, 7, :] = 1
    mask[2, :, 31] = 1
    run_k64_compare(q, k, v, mask, N, d)


@pytest.mark.parametrize("N", [2000, 1985])
def test_bf16_key_blocks_of_64_pairs(N):
    # 64-key blocks are computed two per step: rows with 1, 2 and 3 kept
    # blocks (a last step holding one block), the partial last key block
    # (N = 2000: 16 real keys in block 31; N = 1985: 1 real key) walked in the
    # first half of a step, in the second half and alone, and rows whose walk
    # wraps around from their diagonal block.
    d, Np, H = 128, 2048, 2
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 63)
    mask = np.zeros((H, 16, 32), np.uint8)
    # head 0: the row's own (diagonal) block is walked first
    mask[0, 0, [0]] = 1                       # one block
    mask[0, 1, [2, 3]] = 1                    # one full step
    mask[0, 2, [4, 9, 20]] = 1                # a step and a single block
    mask[0, 3, [31]] = 1                      # the partial block alone
    mask[0, 4, [8, 31]] = 1                   # partial block in the second half
    mask[0, 5, [31, 3]] = 1                   # diagonal 10: walk 31, then 3 (partial block first half)
    mask[0, 6, [12, 13, 31]] = 1              # partial block in a single-block last step
    mask[0, 15, [30, 31]] = 1                 # diagonal 30: 30, 31
    mask[0, 14, [0, 5, 28, 29, 31]] = 1       # odd count with wrap-around
    # head 1: random odd and even counts, last block always kept
    rng = np.random.default_rng(64)
    mask[1] = (rng.random((16, 32)) < 0.2).astype(np.uint8)
    mask[1, :, 31] = 1
    mask[1, 3, :] = 0
    mask[1, 3, 7] = 1
    run_k64_compare(q, k, v, mask, N, d)


def test_bf16_key_blocks_of_64_large_score_jumps():
    # The redo / O-rescale paths with 64-key blocks (magnitudes set per
    # 32-key quarter block, so jumps fall in both halves of a block).
    N, Np, H, d = 2000, 2048, 2, 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 41)
    rng = np.random.default_rng(43)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = (q + 8.0 * u).astype(np.float32)
    g = 12.0 * np.repeat(rng.permutation(64), 32)
    k = (k + g[None, None, :, None] * u).astype(np.float32)
    mask = (rng.random((H, 16, 32)) < 0.5).astype(np.uint8)
    mask[0, 5, :] = 1
    run_k64_compare(q, k, v, mask, N, d)


@pytest.mark.slow
def test_bf16_key_blocks_of_64_wan480_sampled():
    w = syn.WORKLOADS["wan480_25"]
    coarse = syn.workload_mask(w, density=0.375)
    mask = syn.refine_key_blocks(coarse, 0.25, 15)
    q, k, v = syn.video_qkv(w)
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    del q, k, v
    bl = cba.compile(torch.from_numpy(mask).cuda(), block_q=128, block_k=64)
    assert bl.nnz == int(mask.sum())
    scale = cba.default_scale(w.d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, w.N, scale=scale, return_lse=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    rng = np.random.default_rng(16)
    errs = []
    for h, qb in [(0, 0), (w.H - 1, w.nqb - 1)] + [(int(rng.integers(w.H)), int(rng.integers(w.nqb)))
                                                   for _ in range(14)]:
        O, L = oracle.masked_attention_rows(q64, k64, v64, mask, w.N, 128, 64, scale, 0, h, qb)
        rows = slice(qb * 128, (qb + 1) * 128)
        errs.append(np.abs(to_np64(o[0, h, rows]) - O).ravel())
        assert_lse(lse[0, h, rows].cpu().numpy(), L, 1e-3)
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
    print(f"PARITY wan480 128x64 blocks sampled 16 query blocks max_abs={err.max():.3e} mean_abs={err.mean():.3e}")


def run_kv_block_compare(q, k, v, mask, N, d, bk):
    """Whole-tensor parity with 128-row query blocks and bk-key blocks: the
    queries are padded to a multiple of 128 and the keys to a multiple of bk
    (calibatt_sparse_attn_fwd_qk)."""
    npq, npk = q.shape[2], k.shape[2]
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    bl = cba.compile(torch.from_numpy(mask).cuda(), block_q=128, block_k=bk)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = cba.default_scale(d)
    o, lse = cba.sparse_attn_fwd_qk(qd, kd, vd, bl, N, N, scale=scale, return_lse=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    H = q.shape[1]
    O = np.zeros((1, H, npq, d))
    L = np.full((1, H, npq), -np.inf)
    for h in range(H):
        for qb in range(npq // 128):
            O[0, h, qb * 128:(qb + 1) * 128], L[0, h, qb * 128:(qb + 1) * 128] = oracle.masked_attention_rows(
                q64, k64, v64, mask, N, 128, bk, scale, 0, h, qb)
    mx, mn = assert_close(to_np64(o), O, BF16_MAX_ABS, BF16_MEAN_ABS)
    assert_lse(lse.cpu().numpy(), L, 1e-3)
    print(f"PARITY bf16 128x{bk} blocks N={N} d={d} max_abs={mx:.3e} mean_abs={mn:.3e}")


def _kv_inputs(N, bk, d, H, seed):
    npq, npk = -(-N // 128) * 128, -(-N // bk) * bk
    q, _, _ = syn.normal_qkv(1, H, N, npq, d, seed)
    _, k, v = syn.normal_qkv(1, H, N, npk, d, seed + 1)
    return q, k, v, npq // 128, npk // bk


@pytest.mark.parametrize("bk", [80, 96, 144])
@pytest.mark.parametrize("d", [128, 64])
def test_bf16_key_blocks_80_96_144(bk, d):
    # Key blocks of the paper page's Table S6 (B_kv = 80, 96, 144 with
    # B_q = 128): random masks with an empty row, a full row and the padded
    # last key block kept everywhere; ragged N.
    N, H = 1900, 3
    q, k, v, nqb, nkb = _kv_inputs(N, bk, d, H, 71)
    rng = np.random.default_rng(72)
    mask = (rng.random((H, nqb, nkb)) < 0.4).astype(np.uint8)
    mask[0, 4, :] = 0
    mask[1, 7, :] = 1
    mask[2, :, nkb - 1] = 1
    run_kv_block_compare(q, k, v, mask, N, d, bk)


@pytest.mark.parametrize("bk,N", [(144, 934), (80, 1000), (96, 1086)])
def test_bf16_key_blocks_last_block_mostly_padding(bk, N):
    # The last key block holds fewer real keys than the first softmax half's
    # columns (so the second half of that block is all padding), and it is
    # the first block some query tiles walk.
    d, H = 128, 2
    q, k, v, nqb, nkb = _kv_inputs(N, bk, d, H, 81)
    rng = np.random.default_rng(82)
    mask = (rng.random((H, nqb, nkb)) < 0.3).astype(np.uint8)
    mask[:, nqb - 1, :] = 0
    mask[:, nqb - 1, nkb - 1] = 1          # only the padded last block
    mask[0, 0, nkb - 1] = 1
    run_kv_block_compare(q, k, v, mask, N, d, bk)


def test_bf16_key_blocks_80_large_score_jumps():
    # The redo / O-rescale paths with unequal halves (48 + 32 columns).
    N, H, d, bk = 1900, 2, 128, 80
    q, k, v, nqb, nkb = _kv_inputs(N, bk, d, H, 91)
    rng = np.random.default_rng(92)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = (q + 8.0 * u).astype(np.float32)
    g = 12.0 * np.repeat(rng.permutation(k.shape[2] // 16 + 1), 16)[:k.shape[2]]
    k = (k + g[None, None, :, None] * u).astype(np.float32)
    mask = (rng.random((H, nqb, nkb)) < 0.5).astype(np.uint8)
    mask[0, 5, :] = 1
    run_kv_block_compare(q, k, v, mask, N, d, bk)


@pytest.mark.slow
@pytest.mark.parametrize("bk", [80, 96, 144])
def test_bf16_key_blocks_wan480_sampled(bk):
    # The Wan 480p call with the key grid of Table S6 at its reported sparsity
    # (the 128 x 128 structured mask regridded to bk-key blocks).
    w = syn.WORKLOADS["wan480_25"]
    dens = {80: 0.354, 96: 0.359, 144: 0.369}[bk]
    mask = syn.regrid_key_blocks(syn.workload_mask(w, density=dens), w.N, bk, dens, 17)
    q, k, v = syn.video_qkv(w)
    npk = mask.shape[2] * bk
    kp = np.zeros((1, w.H, npk, w.d), np.float32)
    vp = np.zeros_like(kp)
    kp[:, :, :w.N] = k[:, :, :w.N]
    vp[:, :, :w.N] = v[:, :, :w.N]
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(kp)
    v64, vd = bf16_pair(vp)
    del q, k, v, kp, vp
    bl = cba.compile(torch.from_numpy(mask).cuda(), block_q=128, block_k=bk)
    scale = cba.default_scale(w.d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = cba.sparse_attn_fwd_qk(qd, kd, vd, bl, w.N, w.N, scale=scale, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    rng = np.random.default_rng(18)
    errs = []
    for h, qb in [(0, 0), (w.H - 1, w.nqb - 1)] + [(int(rng.integers(w.H)), int(rng.integers(w.nqb)))
                                                   for _ in range(10)]:
        O, _ = oracle.masked_attention_rows(q64, k64, v64, mask, w.N, 128, bk, scale, 0, h, qb)
        errs.append(np.abs(to_np64(o[0, h, qb * 128:(qb + 1) * 128]) - O).ravel())
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
    print(f"PARITY wan480 128x{bk} blocks (density {mask.mean():.3f}) sampled 12 query blocks "
          f"max_abs={err.max():.3e} mean_abs={err.mean():.3e}")


@pytest.mark.parametrize("N", [1, 129])
def test_bf16_degenerate_lengths(N):
    # One real token (the row attends to itself only: O = v_0, LSE = s_00) and
    # a last block holding a single real token; padding rows come back 0 / -inf.
    d, H = 128, 2
    Np = -(-N // 128) * 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 101)
    nb = Np // 128
    mask = np.ones((H, nb, nb), np.uint8)
    run_full_compare(q, k, v, mask, N, 128, "bf16", d)


@pytest.mark.slow
def test_bf16_longest_rows_2048_key_blocks():
    # The longest supported list: 2 048 key blocks per row (262 144 tokens,
    # one head), a ragged end, 1% of the blocks plus the diagonal kept;
    # sampled whole query blocks against the oracle.
    H, d, nb = 1, 128, 2048
    N, Np = nb * 128 - 5, nb * 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 103)
    rng = np.random.default_rng(104)
    mask = (rng.random((H, nb, nb)) < 0.01).astype(np.uint8)
    mask[0, np.arange(nb), np.arange(nb)] = 1
    mask[0, :, nb - 1] = 1
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    v64, vd = bf16_pair(v)
    bl = cba.compile(torch.from_numpy(mask).cuda())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = cba.default_scale(d)
    o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, N, scale=scale, return_lse=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    errs = []
    for qb in (0, 1, 1000, nb - 1):
        O, L = oracle.masked_attention_rows(q64, k64, v64, mask, N, 128, 128, scale, 0, 0, qb)
        rows = slice(qb * 128, (qb + 1) * 128)
        errs.append(np.abs(to_np64(o[0, 0, rows]) - O).ravel())
        assert_lse(lse[0, 0, rows].cpu().numpy(), L, 1e-3)
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
    print(f"PARITY bf16 2048 key blocks per row (N={N}) sampled 4 query blocks max_abs={err.max():.3e} "
          f"mean_abs={err.mean():.3e}")


def test_bf16_forward_replays_in_a_cuda_graph():
    # The forward enqueues only kernels on the caller's stream (descriptors are
    # encoded on the host, nothing is allocated), so a sequence of calls can be
    # captured once and replayed; replays give the eager results bit for bit.
    H, N, Np, d = 3, 2000, 2048, 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 111)
    rng = np.random.default_rng(112)
    masks = (rng.random((3 * H, 16, 16)) < 0.4).astype(np.uint8)
    masks[:, np.arange(16), np.arange(16)] = 1
    _, qd = bf16_pair(q)
    _, kd = bf16_pair(k)
    _, vd = bf16_pair(v)
    bl = cba.compile(torch.from_numpy(masks).cuda())
    eager = [cba.sparse_attn_fwd(qd, kd, vd, bl, N, map_offset=mo) for mo in (0, H, 2 * H)]
    outs = [torch.empty_like(qd) for _ in range(3)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up on the capture stream
        for mo, o in zip((0, H, 2 * H), outs):
            cba.sparse_attn_fwd(qd, kd, vd, bl, N, map_offset=mo, out=o)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for mo, o in zip((0, H, 2 * H), outs):
            cba.sparse_attn_fwd(qd, kd, vd, bl, N, map_offset=mo, out=o)
    for _ in range(2):
        for o in outs:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        for e, o in zip(eager, outs):
            assert torch.equal(e, o)
