"""GPU calibration against the oracle.

Energies are floating point: compared with a tolerance.  Selection, votes and
masks are discrete: fed the GPU's own energies, the oracle must reproduce
them bit for bit.  End to end (oracle energies in float64), masks may differ
only in near-tie rows, whose boundary gap is below 1e-4 of the row's largest
energy.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import synthetic as syn
import oracle

from _util import bf16_pair, fp32_pair

pytestmark = pytest.mark.gpu


def small_inputs(n_inputs, H, grid, d, seed_base=10):
    w = syn.Workload("calib_small", 1, H, grid, d, "bf16", 128, 0.25,
                     {"base": seed_base, "noise_q": 11, "noise_k": 12, "v": 13})
    out = []
    for n in range(n_inputs):
        q, k = syn.video_qkv(w, with_v=False, input_index=n)
        out.append((q[0], k[0]))
    return w, out


@pytest.mark.parametrize("dtype,d,block", [("fp32", 64, 64), ("fp32", 128, 128), ("bf16", 128, 128), ("bf16", 64, 128)])
def test_block_energy(dtype, d, block):
    H = 2
    w, inputs = small_inputs(1, H, syn.VideoGrid(2, 20, 50), d)
    q, k = inputs[0]
    pair = bf16_pair if dtype == "bf16" else fp32_pair
    q64, qd = pair(q)
    k64, kd = pair(k)
    scale = cba.default_scale(d)
    E = cba.block_energy(qd, kd, w.N, block, block, scale=scale).cpu().numpy().astype(np.float64)
    Eo = oracle.block_energy(q64, k64, w.N, block, block, scale)
    nreal = -(-w.N // block)
    rel = np.abs(E - Eo).max()
    print(f"PARITY energy {dtype} d={d} block={block} max_abs={rel:.3e}")
    assert rel <= (1e-5 if dtype == "fp32" else 5e-5), rel
    np.testing.assert_allclose(E[:, :nreal].sum(axis=-1), 1.0, atol=1e-4)


@pytest.mark.parametrize("d,bk", [(128, 64), (128, 80), (128, 96), (128, 144), (64, 80), (64, 144)])
def test_block_energy_key_block_sizes(d, bk):
    # Table S6 key grids (B_kv = 64, 80, 96, 144 against 128-row query
    # blocks): a 128-key score tile meets up to three key blocks; ragged N,
    # so the last key block is partial.
    H = 2
    w, inputs = small_inputs(1, H, syn.VideoGrid(2, 20, 51), d, seed_base=30)
    q, k = inputs[0]
    q64, qd = bf16_pair(q)
    k64, kd = bf16_pair(k)
    scale = cba.default_scale(d)
    E = cba.block_energy(qd, kd, w.N, 128, bk, scale=scale).cpu().numpy().astype(np.float64)
    nke = -(-w.N // bk)
    assert E.shape == (H, w.Np // 128, nke)
    Eo = oracle.block_energy(q64, k64, w.N, 128, bk, scale)
    err = np.abs(E - Eo).max()
    print(f"PARITY energy bf16 d={d} 128x{bk} blocks N={w.N} max_abs={err:.3e}")
    assert err <= 5e-5, err
    nreal = -(-w.N // 128)
    np.testing.assert_allclose(E[:, :nreal].sum(axis=-1), 1.0, atol=1e-4)


def test_calibrate_key_blocks_of_80_drive_the_forward():
    # The Table S6 pipeline at B_kv = 80: calibrate on 80-key blocks, compile,
    # run the forward with keys padded to a multiple of 80.  Discrete stages
    # are bit-exact on the GPU's energies; the forward matches the oracle.
    H, I, bk, d = 2, 3, 80, 128
    w, inputs = small_inputs(I, H, syn.VideoGrid(3, 30, 52), d, seed_base=40)
    pairs = [(bf16_pair(q), bf16_pair(k)) for q, k in inputs]
    qd = [p[0][1] for p in pairs]
    kd = [p[1][1] for p in pairs]
    mv = cba.min_votes_for(0.5, I)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mask, votes, esum = cba.calibrate(qd, kd, w.N, block_k=bk, select_param=0.3, rho=0.5, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    nke = -(-w.N // bk)
    assert mask.shape == (H, w.Np // 128, nke)
    Eg = [cba.block_energy(q, k, w.N, 128, bk).cpu().numpy() for q, k in zip(qd, kd)]
    keeps = [oracle.select_topk(E, 0.3) for E in Eg]
    m_o, v_o, e_o = oracle.vote(np.stack(keeps), mv, np.stack(Eg))
    assert np.array_equal(votes.cpu().numpy(), v_o)
    assert np.array_equal(esum.cpu().numpy(), e_o)
    assert np.array_equal(mask.cpu().numpy(), m_o)
    # forward on input 0 with the calibrated 80-key mask
    npk = nke * bk
    q64, k64 = pairs[0][0][0], pairs[0][1][0]
    rng = np.random.default_rng(41)
    v32 = rng.standard_normal((H, npk, d)).astype(np.float32)
    v32[:, w.N:] = 0.0
    v64, vd = bf16_pair(v32)
    kk = np.zeros((H, npk, d))
    kk[:, :w.N] = k64[:, :w.N]
    kd80 = torch.zeros((1, H, npk, d), dtype=torch.bfloat16, device="cuda")
    kd80[0, :, :w.N] = kd[0][:, :w.N]
    bl = cba.compile(mask, block_q=128, block_k=bk)
    o = cba.sparse_attn_fwd_qk(qd[0][None], kd80, vd[None], bl, w.N, w.N, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    m = mask.cpu().numpy()
    scale = cba.default_scale(d)
    err = 0.0
    for h, qb in ((0, 0), (0, 7), (1, 3), (1, w.Np // 128 - 1)):
        ref, _ = oracle.masked_attention_rows(q64[None], kk[None], v64[None], m, w.N, 128, bk, scale, 0, h, qb)
        got = o[0, h, qb * 128:(qb + 1) * 128].float().cpu().numpy()
        real = min(128, w.N - qb * 128)
        err = max(err, np.abs(got[:real] - ref[:real]).max())
    print(f"PARITY calibrate+forward 128x{bk} blocks max_abs={err:.3e}")
    assert err <= 2e-2, err


def test_select_vote_finalize_bit_exact():
    rng = np.random.default_rng(4)
    H, nqb, nkb, I = 3, 9, 37, 5
    Es = [rng.random((H, nqb, nkb)).astype(np.float32) for _ in range(I)]
    Es[0][0, 0, 5] = Es[0][0, 0, 6]                      # exact tie
    Es[1][1, 2, :] = 0.25                                # all ties
    for mode, param in ((cba.SELECT_TOPK, 0.25), (cba.SELECT_ENERGY, 0.3), (cba.SELECT_ENERGY, 0.0)):
        votes = torch.zeros((H, nqb, nkb), dtype=torch.int32, device="cuda")
        esum = torch.zeros((H, nqb, nkb), dtype=torch.float32, device="cuda")
        keeps = []
        for E in Es:
            cba.select_vote(torch.from_numpy(E).cuda(), mode, param, votes, esum)
            keeps.append(oracle.select_topk(E, param) if mode == cba.SELECT_TOPK else oracle.select_energy(E, param))
        for mv in (1, 3, 5):
            mask = cba.finalize_mask(votes, esum, mv)
            m_o, v_o, e_o = oracle.vote(np.stack(keeps), mv, np.stack(Es))
            assert np.array_equal(votes.cpu().numpy(), v_o)
            assert np.array_equal(esum.cpu().numpy(), e_o)
            assert np.array_equal(mask.cpu().numpy(), m_o)


def near_tie_rows(E, k):
    """Rows whose k-th and (k+1)-th energies are closer than 1e-4 of the row maximum."""
    s = -np.sort(-E, axis=-1)
    gap = s[..., k - 1] - s[..., k]
    return gap < 1e-4 * s[..., 0]


def test_calibration_resumes_from_saved_state(tmp_path):
    # Votes and energy sums add up over inputs (Figure 3(b): a block's count
    # over the calibration prompts): a calibration saved after 3 of 6 inputs,
    # reloaded and continued with the other 3 (inputs_before = 3), ends with
    # the votes, energy sums and mask of one 6-input pass, bit for bit.  The
    # threshold counts all 6 inputs: ceil(0.5 * 6) = 3 votes, not 2.
    H, I = 2, 6
    w, inputs = small_inputs(I, H, syn.VideoGrid(2, 20, 50), 128, seed_base=50)
    qd = [bf16_pair(q)[1] for q, _ in inputs]
    kd = [bf16_pair(k)[1] for _, k in inputs]
    mask1, votes1, esum1 = cba.calibrate(qd, kd, w.N, select_param=0.3, rho=0.5)
    m_half, v_half, e_half = cba.calibrate(qd[:3], kd[:3], w.N, select_param=0.3, rho=0.5, finalize=False)
    assert m_half is None
    p = tmp_path / "calib.npz"
    cba.save_calibration(p, v_half, e_half, 3, select_param=0.3, rho=0.5)
    v, e, n, meta = cba.load_calibration(p, device="cuda")
    mask2, votes2, esum2 = cba.calibrate(qd[3:], kd[3:], w.N, select_param=meta["select_param"], rho=meta["rho"],
                                         votes=v, energy_sum=e, inputs_before=n)
    assert torch.equal(votes2, votes1)
    assert torch.equal(esum2, esum1)
    assert torch.equal(mask2, mask1)
    assert torch.equal(mask1, cba.finalize_mask(votes1, esum1, 3))


def test_calibrate_small_end_to_end():
    H, I = 2, 4
    w, inputs = small_inputs(I, H, syn.VideoGrid(3, 30, 52), 128)
    nb = w.Np // 128
    pairs = [(bf16_pair(q), bf16_pair(k)) for q, k in inputs]
    qd = [p[0][1] for p in pairs]
    kd = [p[1][1] for p in pairs]
    mv = cba.min_votes_for(0.5, I)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mask, votes, esum = cba.calibrate(qd, kd, w.N, select_param=0.25, rho=0.5, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # discrete stages on the GPU's energies: bit-exact
    Eg = [cba.block_energy(q, k, w.N).cpu().numpy() for q, k in zip(qd, kd)]
    keeps = [oracle.select_topk(E, 0.25) for E in Eg]
    m_o, v_o, e_o = oracle.vote(np.stack(keeps), mv, np.stack(Eg))
    assert np.array_equal(votes.cpu().numpy(), v_o)
    assert np.array_equal(esum.cpu().numpy(), e_o)
    assert np.array_equal(mask.cpu().numpy(), m_o)
    # end to end against float64 energies: differences only in near-tie rows
    Eo = [oracle.block_energy(p[0][0], p[1][0], w.N, 128, 128, cba.default_scale(128)) for p in pairs]
    k = oracle.topk_count(0.25, nb)
    keeps64 = [oracle.select_topk(E, 0.25) for E in Eo]
    m64, _, _ = oracle.vote(np.stack(keeps64), mv, np.stack(Eo))
    tie = np.zeros((H, nb), bool)
    for E in Eo:
        tie |= near_tie_rows(E, k)
    diff_rows = (mask.cpu().numpy() != m64).any(axis=-1)
    print(f"PARITY calibrate rows_differing={int(diff_rows.sum())} near_tie_rows={int(tie.sum())} of {tie.size}")
    assert not (diff_rows & ~tie).any()
    # the compiled calibrated mask drives the forward kernel
    bl = cba.compile(mask)
    assert bl.nnz == int(mask.sum().item())


@pytest.mark.slow
def test_calibrate_wan_config_full_size_against_float64_oracle():
    # The calibration workload at full size: 8 Wan 480p inputs (40 heads,
    # 32 760 tokens).  For 4 heads the float64 oracle scores every input: the
    # GPU's energies must match element by element, and the masks that the
    # oracle's selection and vote build from its own float64 energies may
    # differ from the GPU's masks only in near-tie rows.
    from _oracle_pool import block_energies
    w = syn.WORKLOADS["wan480_25"]
    I, heads = 8, [0, 13, 26, 39]
    scale = cba.default_scale(w.d)
    qd, kd, jobs = [], [], []
    for n in range(I):
        q, k = syn.video_qkv(w, with_v=False, input_index=n)
        q64, qg = bf16_pair(q[0])
        k64, kg = bf16_pair(k[0])
        qd.append(qg)
        kd.append(kg)
        jobs += [(q64[h:h + 1].copy(), k64[h:h + 1].copy(), w.N, 128, scale) for h in heads]
        del q, k, q64, k64
    mask, votes, esum = cba.calibrate(qd, kd, w.N, select_param=0.25, rho=0.5)
    Eg = np.stack([cba.block_energy(q, k, w.N)[heads].cpu().numpy() for q, k in zip(qd, kd)])
    mask_g = mask[heads].cpu().numpy()
    del qd, kd
    torch.cuda.empty_cache()
    Eo = np.stack(block_energies(jobs)).reshape(I, len(heads), w.nqb, w.nqb)
    err = np.abs(Eg.astype(np.float64) - Eo)
    print(f"PARITY energy wan480 8 inputs x {len(heads)} heads: max_abs={err.max():.3e} mean_abs={err.mean():.3e}")
    assert err.max() <= 5e-5
    k = oracle.topk_count(0.25, w.nqb)
    keeps = [oracle.select_topk(E, 0.25) for E in Eo]
    m64, _, _ = oracle.vote(np.stack(keeps), oracle.min_votes_for(0.5, I), Eo)
    tie = np.zeros((len(heads), w.nqb), bool)
    close = np.zeros((len(heads), w.nqb), bool)
    for E in Eo:
        tie |= near_tie_rows(E, k)
        # rows whose k-th and (k+1)-th energies are closer than twice the
        # measured GPU energy error: the only rows whose selection the
        # float32 energies can change
        srt = -np.sort(-E, axis=-1)
        close |= (srt[..., k - 1] - srt[..., k]) < 2 * err.max()
    diff_rows = (mask_g != m64).any(axis=-1)
    print(f"PARITY calibrate wan480 end to end: rows_differing={int(diff_rows.sum())} of {tie.size}; rows within "
          f"2x the energy error of a tie={int(close.sum())}; near-tie rows by the 1e-4 relative rule={int(tie.sum())}")
    assert not (diff_rows & ~close).any()


@pytest.mark.slow
def test_calibrate_wan_config_subset():
    # 8 calibration inputs of the Wan 480p shape; the oracle's discrete stages
    # run on the GPU's energies for every head.
    w = syn.WORKLOADS["wan480_25"]
    I = 8
    qd, kd = [], []
    for n in range(I):
        q, k = syn.video_qkv(w, with_v=False, input_index=n)
        qd.append(bf16_pair(q[0])[1])
        kd.append(bf16_pair(k[0])[1])
        del q, k
    mask, votes, esum = cba.calibrate(qd, kd, w.N, select_param=0.25, rho=0.5)
    Eg = [cba.block_energy(q, k, w.N).cpu().numpy() for q, k in zip(qd, kd)]
    keeps = [oracle.select_topk(E, 0.25) for E in Eg]
    m_o, v_o, _ = oracle.vote(np.stack(keeps), 4, np.stack(Eg))
    assert np.array_equal(votes.cpu().numpy(), v_o)
    assert np.array_equal(mask.cpu().numpy(), m_o)
    np.testing.assert_allclose(np.stack(Eg)[:, :, :, :].sum(axis=-1), 1.0, atol=2e-3)
    print(f"PARITY calibrate-wan480 8 inputs: votes and masks bit-exact; mask density {float(mask.float().mean()):.4f}")
    # time of one calibration pass (8 inputs: energies, selection, votes, mask) on the device
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    cba.calibrate(qd, kd, w.N, select_param=0.25, rho=0.5)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    flops = I * 2 * 2 * w.N * w.N * w.d * w.H   # two QK^T passes per input
    print(f"TIMING calibrate-wan480 8 inputs: {ms:.1f} ms, energy passes {flops / ms / 1e9:.1f} TFLOP/s")


def test_sharded_calibration_single_rank_matches_calibrate():
    # Calibration sharded by input, run as one NCCL rank on one GPU: the
    # gather, per-input selection, votes and threshold must give exactly the
    # single-call calibration's mask, votes and energy sums.
    import os
    import socket
    import torch.distributed as dist
    from block_sparse_attention_cross_b200.sharded import calibrate_sharded
    H = 2
    w, inputs = small_inputs(4, H, syn.VideoGrid(3, 20, 50), 128)
    qd = [bf16_pair(q)[1] for q, _ in inputs]
    kd = [bf16_pair(k)[1] for _, k in inputs]
    mask1, votes1, esum1 = cba.calibrate(qd, kd, w.N, select_param=0.25, rho=0.5)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        mask2, votes2, esum2 = calibrate_sharded(qd, kd, w.N, select_param=0.25, rho=0.5)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(votes1, votes2)
    assert torch.equal(esum1, esum2)
    assert torch.equal(mask1, mask2)


def test_energy_schedule_per_timestep():
    # One calibration per step with its own energy threshold (a schedule the
    # caller supplies: the pages plot one but print no values); every step's
    # mask equals the oracle's selection and vote on that step's GPU energies.
    H = 2
    steps = []
    for t in range(3):
        w, inputs = small_inputs(3, H, syn.VideoGrid(2, 20, 50), 128, seed_base=20 + t)
        steps.append(([bf16_pair(q)[1] for q, _ in inputs], [bf16_pair(k)[1] for _, k in inputs]))
    eps = lambda t, T: 0.05 + 0.3 * t / max(1, T - 1)
    masks = cba.calibrate_schedule(steps, w.N, eps, rho=0.5)
    assert masks.shape[0] == 3
    for t, (qd, kd) in enumerate(steps):
        Eg = [cba.block_energy(q, k, w.N).cpu().numpy() for q, k in zip(qd, kd)]
        keeps = [oracle.select_energy(E, eps(t, 3)) for E in Eg]
        m_o, _, _ = oracle.vote(np.stack(keeps), oracle.min_votes_for(0.5, 3), np.stack(Eg))
        assert np.array_equal(masks[t].cpu().numpy(), m_o)
    dens = [float(m.float().mean()) for m in masks]
    print(f"PARITY energy schedule: 3 steps, densities {', '.join(f'{x:.3f}' for x in dens)}, masks bit-exact")
