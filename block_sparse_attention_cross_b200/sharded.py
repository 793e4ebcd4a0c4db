"""Calibration sharded by input across ranks (one process per GPU).

CalibAtt's calibration (paper page, Figure 5(a) and Figure 3(b)) scores every
calibration input, keeps the top key blocks per query block and keeps a block
when enough inputs agree.  Scoring an input -- the dense block energies, two
QK^T passes over the whole sequence -- is where the time goes, and inputs are
independent, so ranks split the inputs: each rank computes the energies of
its own inputs on its GPU, the per-input energies are all-gathered over the
process group (NCCL over NVLink between GPUs; gloo for CPU tests), and every
rank then runs selection, voting and the agreement threshold over all inputs
in global input order with the same kernels as a single-GPU calibration.
Every rank therefore ends with the same mask, bit-identical to calibrating
all inputs on one GPU (the vote counts are integers and the float32 energy
sums are accumulated in the same order).

Ranks hold contiguous input ranges in rank order (rank 0 the first inputs).
"""

from __future__ import annotations

import torch


def gather_in_order(local, group=None):
    """All-gathers each rank's list of equally shaped tensors; returns the
    concatenation in rank order (rank 0's tensors first).  Ranks may hold
    different counts, but at least one tensor each: every rank takes the
    shape of the padded exchange from its own first tensor (ValueError
    otherwise)."""
    import torch.distributed as dist
    if not local:
        raise ValueError("every rank needs at least one tensor")
    world = dist.get_world_size(group)
    dev = local[0].device
    counts = torch.tensor([len(local)], dtype=torch.int64, device=dev)
    all_counts = [torch.zeros_like(counts) for _ in range(world)]
    dist.all_gather(all_counts, counts, group=group)
    all_counts = [int(c.item()) for c in all_counts]
    n_max = max(all_counts)
    stack = torch.stack(list(local) + [torch.zeros_like(local[0])] * (n_max - len(local)))
    parts = [torch.empty_like(stack) for _ in range(world)]
    dist.all_gather(parts, stack.contiguous(), group=group)
    out = []
    for r in range(world):
        out.extend(parts[r][i] for i in range(all_counts[r]))
    return out


def calibrate_sharded(q_local, k_local, N, group=None, block_q=128, block_k=128, scale=None, select_mode=None,
                      select_param=0.25, rho=0.5, min_votes=None):
    """Calibration over the inputs of all ranks; q_local / k_local: this
    rank's inputs ([H, Np, d] CUDA tensors, at least one per rank).

    Returns (mask, votes, energy_sum) -- identical on every rank."""
    import block_sparse_attention_cross_b200 as cba
    if select_mode is None:
        select_mode = cba.SELECT_TOPK
    if len(q_local) != len(k_local) or not q_local:
        raise ValueError("need the same non-zero number of q and k tensors on every rank")
    energies = [cba.block_energy(q, k, N, block_q=block_q, block_k=block_k, scale=scale)
                for q, k in zip(q_local, k_local)]
    all_e = gather_in_order(energies, group)
    H, nqb, nkb = all_e[0].shape
    dev = all_e[0].device
    votes = torch.zeros((H, nqb, nkb), dtype=torch.int32, device=dev)
    esum = torch.zeros((H, nqb, nkb), dtype=torch.float32, device=dev)
    for E in all_e:
        cba.select_vote(E.contiguous(), select_mode, select_param, votes, esum)
    mv = cba.min_votes_for(rho, len(all_e)) if min_votes is None else int(min_votes)
    mask = cba.finalize_mask(votes, esum, mv)
    return mask, votes, esum
