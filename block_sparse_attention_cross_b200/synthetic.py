"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws inputs only: random tensors, bf16 rounding of those tensors,
and block masks with the structures the CalibAtt paper page shows in its
figures (frame-diagonal blocks and within-frame row repetition, Figures 2
and 4).  It holds none of the method's arithmetic (no softmax, no energies, no
selection, no voting, no compilation), so both the CUDA path and the CPU
oracle can consume its output without sharing any of the method.

No model weights, prompts or benchmark items are involved: the workloads of
the paper page (Wan 2.1 14B, Mochi 1 video generations) enter only through
their attention shapes.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np


def _threads():
    return max(1, min(16, len(os.sched_getaffinity(0))))

# --------------------------------------------------------------------------
# bf16 helpers (round-to-nearest-even on the float32 bit pattern)
# --------------------------------------------------------------------------


def _bf16_bits_chunk(x):
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def f32_to_bf16_bits(x):
    """Round float32 values to bf16 (nearest even); returns uint16 bit patterns.

    Large arrays are rounded in chunks on a thread pool (numpy releases the
    GIL); the result does not depend on the chunking.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1)
    if flat.size < (1 << 22):
        return _bf16_bits_chunk(flat).reshape(x.shape)
    out = np.empty(flat.size, dtype=np.uint16)
    step = 1 << 21
    starts = range(0, flat.size, step)

    def work(i):
        out[i:i + step] = _bf16_bits_chunk(flat[i:i + step])

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, starts))
    return out.reshape(x.shape)


def bf16_bits_to_f32(bits):
    """Exact float32 values of bf16 bit patterns."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def round_to_bf16(x):
    """float32 array of the bf16-rounded values of ``x``."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# --------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class VideoGrid:
    frames: int
    rows: int
    cols: int
    text_tokens: int = 0

    @property
    def video_tokens(self):
        return self.frames * self.rows * self.cols

    @property
    def n_tokens(self):
        return self.video_tokens + self.text_tokens


def padded(n, block):
    return ((n + block - 1) // block) * block


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: VideoGrid
    d: int
    dtype: str              # "bf16" or "fp32"
    block: int
    density: float
    seeds: dict = field(default_factory=dict)

    @property
    def N(self):
        return self.grid.n_tokens

    @property
    def Np(self):
        return padded(self.N, self.block)

    @property
    def nqb(self):
        return self.Np // self.block


WORKLOADS = {
    # 4 frames x 16 x 16 = 1024 tokens, fp32, 64 x 64 blocks, 50% random mask
    "tiny_fp32": Workload("tiny_fp32", 1, 2, VideoGrid(4, 16, 16), 64, "fp32", 64, 0.5,
                          {"data": 1, "mask": 2}),
    # Wan 2.1 14B 480p attention call: 21 x 30 x 52 = 32760 tokens -> 32768
    "wan480_25": Workload("wan480_25", 1, 40, VideoGrid(21, 30, 52), 128, "bf16", 128, 0.25,
                          {"base": 10, "noise_q": 11, "noise_k": 12, "v": 13, "mask": 14}),
    # Wan 2.1 14B 720p: 21 x 45 x 80 = 75600 tokens -> 75648
    "wan720_20": Workload("wan720_20", 1, 40, VideoGrid(21, 45, 80), 128, "bf16", 128, 0.20,
                          {"base": 20, "noise_q": 21, "noise_k": 22, "v": 23, "mask": 24}),
    # Mochi 1: 28 x 30 x 53 = 44520 video tokens + 256 text tokens = 44776 -> 44800
    "mochi_20": Workload("mochi_20", 1, 24, VideoGrid(28, 30, 53, text_tokens=256), 128, "bf16", 128, 0.20,
                         {"base": 30, "noise_q": 31, "noise_k": 32, "v": 33, "mask": 34}),
}


# --------------------------------------------------------------------------
# Dense tensors
# --------------------------------------------------------------------------


def normal_qkv(B, H, N, Np, d, seed):
    """Q, K, V ~ N(0, 1) float32 [B, H, Np, d]; padding rows (>= N) are 0."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        x = np.zeros((B, H, Np, d), dtype=np.float32)
        x[:, :, :N] = rng.standard_normal((B, H, N, d), dtype=np.float32)
        out.append(x)
    return tuple(out)


def _token_coords(grid: VideoGrid):
    t = np.arange(grid.video_tokens)
    f = t // (grid.rows * grid.cols)
    y = (t // grid.cols) % grid.rows
    x = t % grid.cols
    return f, y, x


def video_qk_base(grid: VideoGrid, H, d, seed, rank=16, alpha=1.0, jitter=0.0, jitter_seed=None, row_scale=None):
    """Shared low-rank frame/row/column structure: [H, video_tokens, d] float32.

    base[h, t] = alpha * (F[h, f(t)] + s_h Y[h, y(t)] + X[h, x(t)]) @ W[h], with
    F, Y, X ~ N(0, 1) of width ``rank`` and W ~ N(0, 1/rank); s_h =
    ``row_scale[h]`` (1 when not given: heads whose s_h is small see nearly the
    same tokens on every spatial row of a frame).  ``jitter`` adds
    N(0, jitter^2) to F, Y and X from ``jitter_seed`` (per calibration input).
    """
    rng = np.random.default_rng(seed)
    F = rng.standard_normal((H, grid.frames, rank))
    Y = rng.standard_normal((H, grid.rows, rank))
    X = rng.standard_normal((H, grid.cols, rank))
    W = rng.standard_normal((H, rank, d)) / math.sqrt(rank)
    if jitter:
        jr = np.random.default_rng(jitter_seed)
        F = F + jitter * jr.standard_normal(F.shape)
        Y = Y + jitter * jr.standard_normal(Y.shape)
        X = X + jitter * jr.standard_normal(X.shape)
    f, y, x = _token_coords(grid)
    base = np.empty((H, grid.video_tokens, d), dtype=np.float32)

    rs = np.ones(H) if row_scale is None else np.asarray(row_scale, np.float64)

    def head(h):
        lat = F[h][f] + rs[h] * Y[h][y] + X[h][x]
        base[h] = (alpha * (lat @ W[h])).astype(np.float32)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(head, range(H)))
    return base


def video_qkv(w: Workload, noise=0.1, with_v=True, input_index=None, jitter=0.05, row_scale=None):
    """Q, K (and V) float32 [B, H, Np, d] for a video-shaped workload.

    Q and K share the low-rank base and get independent N(0, noise^2) noise;
    text tokens (if any) and V are N(0, 1); padding rows are 0.  With
    ``input_index`` = n the base gets a per-input jitter and the noise comes
    from seeds derived from 100 + n (calibration inputs).  Every (tensor,
    batch, head) slice draws from its own stream, seeded by (seed, b, h), so
    the slices are filled in parallel and the values do not depend on the
    thread count.  ``row_scale``: per-head weight of the spatial-row term of
    the base (see :func:`video_qk_base`).
    """
    g = w.grid
    s = w.seeds
    if input_index is None:
        base = video_qk_base(g, w.H, w.d, s["base"], row_scale=row_scale)
        sq, sk = [s["noise_q"]], [s["noise_k"]]
    else:
        base = video_qk_base(g, w.H, w.d, s["base"], jitter=jitter, jitter_seed=100 + input_index,
                             row_scale=row_scale)
        sq, sk = [100 + input_index, 1], [100 + input_index, 2]
    sv = [s.get("v", 0)]
    Nv, N, Np = g.video_tokens, w.N, w.Np
    q = np.zeros((w.B, w.H, Np, w.d), dtype=np.float32)
    k = np.zeros_like(q)
    v = np.zeros_like(q) if with_v else None

    def plane(bh):
        b, h = divmod(bh, w.H)
        for x, seed in ((q, sq), (k, sk)):
            r = np.random.default_rng(seed + [b, h])
            x[b, h, :Nv] = base[h] + noise * r.standard_normal((Nv, w.d), dtype=np.float32)
            if N > Nv:
                x[b, h, Nv:N] = r.standard_normal((N - Nv, w.d), dtype=np.float32)
        if v is not None:
            v[b, h, :N] = np.random.default_rng(sv + [b, h]).standard_normal((N, w.d), dtype=np.float32)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(plane, range(w.B * w.H)))
    if not with_v:
        return q, k
    return q, k, v


# --------------------------------------------------------------------------
# Block masks
# --------------------------------------------------------------------------


def random_block_mask(H, nqb, nkb, n_offdiag, seed):
    """Per head: the diagonal blocks plus exactly ``n_offdiag`` off-diagonal blocks, uniform without replacement."""
    rng = np.random.default_rng(seed)
    mask = np.zeros((H, nqb, nkb), dtype=np.uint8)
    diag = np.arange(min(nqb, nkb))
    off = np.array([i * nkb + j for i in range(nqb) for j in range(nkb) if i != j], dtype=np.int64)
    for h in range(H):
        mask[h, diag, diag] = 1
        pick = rng.choice(off, size=n_offdiag, replace=False)
        mask[h].reshape(-1)[pick] = 1
    return mask


def structured_block_mask(n_maps, nqb, nkb, density, seed, row_width, frame_tokens, block=128,
                          band=3, period=None, forced_cols=(), local_frames=4):
    """Block masks with frame-diagonal and row-periodic structure, exact density.

    Per map: the period P_b = lcm(row_width, block) / block (query blocks after
    which the spatial-row grid and the block grid line up again) unless given.
    Each phase r < P_b draws a set of relative offsets: 0, the band
    |delta| <= ``band``, offsets near multiples of the frame stride
    ``frame_tokens / block`` (the same spatial position in up to
    ``local_frames`` neighbouring frames), then random offsets inside that
    neighbourhood up to the per-row budget round(density * nkb).  Row qb keeps
    qb + delta for the offsets of phase qb mod P_b (so interior rows of one
    phase are exact translates of each other), plus the diagonal and
    ``forced_cols``.  Rows cut short by the sequence edges are topped up with
    random nearby blocks, and a last random adjustment hits
    round(density * nqb * nkb) kept blocks exactly.  ``density`` may be a
    scalar or one value per map.
    """
    rng = np.random.default_rng(seed)
    if period is None:
        period = math.lcm(int(row_width), int(block)) // int(block)
    stride = frame_tokens / block
    dens = np.broadcast_to(np.asarray(density, dtype=np.float64), (n_maps,))
    forced_cols = np.asarray(sorted(set(int(c) for c in forced_cols)), dtype=np.int64)
    masks = np.zeros((n_maps, nqb, nkb), dtype=np.uint8)
    for m in range(n_maps):
        target = int(round(dens[m] * nqb * nkb))
        per_row = min(nkb, max(1, int(round(dens[m] * nkb))))
        w_local = max(band + 1, int(round(local_frames * stride)), per_row)
        mk = masks[m]
        phases = []
        for r in range(period):
            offs = [0]
            for dlt in range(1, band + 1):
                offs += [dlt, -dlt]
            for mult in range(1, local_frames + 1):
                for sgn in (1, -1):
                    c = int(round(sgn * mult * stride))
                    for e in (0, 1 if rng.random() < 0.5 else -1):
                        if c + e not in offs:
                            offs.append(c + e)
            offs = offs[:per_row]
            taken = set(offs)
            pool = [x for x in range(-w_local, w_local + 1) if x not in taken]
            extra = per_row - len(offs)
            if extra > 0:
                offs += [int(x) for x in rng.choice(pool, size=min(extra, len(pool)), replace=False)]
            phases.append(np.asarray(offs, dtype=np.int64))
        protected = np.zeros((nqb, nkb), dtype=bool)
        diag = np.arange(min(nqb, nkb))
        protected[diag, diag] = True
        if forced_cols.size:
            protected[:, forced_cols] = True
        for qb in range(nqb):
            cols = qb + phases[qb % period]
            cols = cols[(cols >= 0) & (cols < nkb)]
            mk[qb, cols] = 1
            mk[qb, protected[qb]] = 1
            short = per_row - int(mk[qb].sum())
            if short > 0:
                lo, hi = max(0, qb - w_local), min(nkb, qb + w_local + 1)
                free = np.flatnonzero(mk[qb, lo:hi] == 0) + lo
                if free.size < short:
                    free = np.flatnonzero(mk[qb] == 0)
                mk[qb, rng.choice(free, size=min(short, free.size), replace=False)] = 1
        cur = int(mk.sum())
        if cur < target:
            free = np.flatnonzero(mk.reshape(-1) == 0)
            add = rng.choice(free, size=min(target - cur, free.size), replace=False)
            mk.reshape(-1)[add] = 1
        elif cur > target:
            removable = np.flatnonzero((mk.reshape(-1) == 1) & ~protected.reshape(-1))
            drop = rng.choice(removable, size=min(cur - target, removable.size), replace=False)
            mk.reshape(-1)[drop] = 0
    return masks


def workload_mask(w: Workload, density=None, n_maps=None, seed=None):
    """The block mask a workload is timed with (per head), exact density."""
    dens = w.density if density is None else density
    n_maps = w.H if n_maps is None else n_maps
    seed = w.seeds.get("mask", 0) if seed is None else seed
    nkb = w.Np // w.block
    if w.name == "tiny_fp32":
        n_off = int(round(dens * w.nqb * nkb)) - min(w.nqb, nkb)
        return random_block_mask(n_maps, w.nqb, nkb, n_off, seed)
    g = w.grid
    forced = ()
    period = None
    if g.text_tokens:
        first_text_block = g.video_tokens // w.block
        forced = range(first_text_block, nkb)
        period = 13
    return structured_block_mask(n_maps, w.nqb, nkb, dens, seed, g.cols, g.rows * g.cols,
                                 block=w.block, period=period, forced_cols=forced)


def refine_key_blocks(mask, density, seed):
    """A mask on a key grid twice as fine (key blocks of 64 for query blocks of
    128): each kept 128-key block contributes its two 64-key halves, both
    halves of the query's own (diagonal) block are always kept, and the other
    halves are kept at random to hit round(density * nqb * 2 nkb) exactly.
    ``mask`` [n_maps, nqb, nkb] should keep more than ``density`` of its
    blocks.  Returns uint8 [n_maps, nqb, 2 nkb].
    """
    rng = np.random.default_rng(seed)
    n_maps, nqb, nkb = mask.shape
    out = np.zeros((n_maps, nqb, 2 * nkb), dtype=np.uint8)
    for m in range(n_maps):
        cand = np.repeat(mask[m] != 0, 2, axis=1)
        diag = np.zeros_like(cand)
        q = np.arange(nqb)
        diag[q, np.minimum(2 * q, 2 * nkb - 1)] = True
        diag[q, np.minimum(2 * q + 1, 2 * nkb - 1)] = True
        target = int(round(density * nqb * 2 * nkb))
        keep = diag.copy()
        rest = np.flatnonzero(cand & ~diag)
        need = max(0, target - int(keep.sum()))
        if need > rest.size:
            raise ValueError("the coarse mask keeps too few blocks for this density")
        keep.ravel()[rng.choice(rest, size=need, replace=False)] = True
        out[m] = keep
    return out


def sweep_masks(w: Workload, layers=40, timesteps=3, seed=1000, lo=0.1, hi=0.6):
    """Mask dictionary of a denoising-step sweep: one structured mask per (layer, timestep, head).

    Map id = (layer * timesteps + t) * H + head; map m has density ~ U(lo, hi)
    (one draw per map from ``seed``) and its own structure seed ``seed + m``.
    """
    n_maps = layers * timesteps * w.H
    dens = np.random.default_rng(seed).uniform(lo, hi, n_maps)
    g = w.grid
    out = np.empty((n_maps, w.nqb, w.nqb), dtype=np.uint8)
    for m in range(n_maps):
        out[m] = structured_block_mask(1, w.nqb, w.nqb, dens[m], seed + m, g.cols, g.rows * g.cols,
                                       block=w.block)[0]
    return out



def regrid_key_blocks(mask, N, block_k, density, seed, block=128):
    """The same mask on a grid of ``block_k``-token key blocks (query blocks stay
    ``block`` tokens): a new key block is kept when it overlaps a kept block of
    ``mask`` [n_maps, nqb, nkb]; the blocks overlapping the query block's own
    tokens are always kept; then blocks are dropped (or added) at random to hit
    round(density * nqb * nkb') exactly, nkb' = ceil(N / block_k).
    Returns uint8 [n_maps, nqb, nkb'].
    """
    rng = np.random.default_rng(seed)
    n_maps, nqb, nkb = mask.shape
    nkb2 = -(-N // block_k)
    lo = np.arange(nkb2) * block_k
    hi = np.minimum(lo + block_k, N)
    # coarse block c covers tokens [c block, (c + 1) block): overlap matrix [nkb2, nkb]
    c_lo = np.arange(nkb) * block
    over = (lo[:, None] < c_lo[None, :] + block) & (hi[:, None] > c_lo[None, :])
    q_lo = np.arange(nqb) * block
    own = (lo[None, :] < q_lo[:, None] + block) & (hi[None, :] > q_lo[:, None])   # [nqb, nkb2]
    target = int(round(density * nqb * nkb2))
    out = np.zeros((n_maps, nqb, nkb2), dtype=np.uint8)
    for m in range(n_maps):
        keep = ((mask[m] != 0).astype(np.int64) @ over.T.astype(np.int64)) > 0
        keep |= own
        cur = int(keep.sum())
        if cur > target:
            removable = np.flatnonzero(keep.ravel() & ~own.ravel())
            drop = rng.choice(removable, size=min(cur - target, removable.size), replace=False)
            keep.ravel()[drop] = False
        elif cur < target:
            free = np.flatnonzero(~keep.ravel())
            keep.ravel()[rng.choice(free, size=min(target - cur, free.size), replace=False)] = True
        out[m] = keep
    return out
