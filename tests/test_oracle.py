"""Pins for the CPU oracle, none of which re-types its formulas.

Each test compares the oracle with something fixed independently of it: a
textbook library routine (torch scaled_dot_product_attention on CPU in
float64), pure-Python brute force, closed forms, or invariants that the
CalibAtt paper page fixes (Figure 3(b): a block kept for every prompt is
always computed).  The cases are chosen so that a plausible slip -- a swapped
block index, a dropped scale, a missing padding rule, an off-by-one in the
top-k count, a wrong tie-break, a wrong vote comparison -- fails one of them.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(1234)


def sdpa64(q, k, v, scale):
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], scale=scale)[0].numpy()


# ----------------------------------------------------------------- O1 attention

def test_all_ones_mask_is_dense_sdpa():
    B, H, N, Np, d, blk = 2, 3, 45, 48, 16, 8
    q, k, v = (RNG.standard_normal((B, H, Np, d)) for _ in range(3))
    mask = np.ones((H, Np // blk, Np // blk), np.uint8)
    scale = 0.37
    O, L = oracle.masked_attention(q, k, v, mask, N, blk, blk, scale)
    for b in range(B):
        for h in range(H):
            ref = sdpa64(q[b, h, :N], k[b, h, :N], v[b, h, :N], scale)
            np.testing.assert_allclose(O[b, h, :N], ref, atol=1e-12, rtol=0)
            s = scale * q[b, h, :N] @ k[b, h, :N].T
            lse_ref = np.array([math.log(math.fsum(math.exp(x) for x in row)) for row in s])
            np.testing.assert_allclose(L[b, h, :N], lse_ref, atol=1e-12, rtol=0)
    assert np.all(O[:, :, N:] == 0) and np.all(np.isneginf(L[:, :, N:]))


def brute_attention(q, k, v, mask, N, bq, bk, scale):
    """Pure-Python loops; independent of numpy's linear algebra."""
    Np, d = len(q), len(q[0])
    O = [[0.0] * d for _ in range(Np)]
    L = [float("-inf")] * Np
    for i in range(N):
        js = [j for j in range(N) if mask[i // bq][j // bk]]
        if not js:
            continue
        s = [scale * math.fsum(q[i][t] * k[j][t] for t in range(d)) for j in js]
        m = max(s)
        p = [math.exp(x - m) for x in s]
        z = math.fsum(p)
        for t in range(d):
            O[i][t] = math.fsum(p[a] * v[j][t] for a, j in enumerate(js)) / z
        L[i] = m + math.log(z)
    return np.array(O), np.array(L)


@pytest.mark.parametrize("N,Np,bq,bk", [(13, 16, 4, 4), (30, 32, 8, 4), (7, 8, 4, 8)])
def test_brute_force_small(N, Np, bq, bk):
    H, d = 2, 5
    q, k, v = (RNG.standard_normal((1, H, Np, d)) for _ in range(3))
    mask = (RNG.random((H, Np // bq, Np // bk)) < 0.5).astype(np.uint8)
    mask[0, 0, :] = 0           # an empty query-block row
    scale = 0.8
    O, L = oracle.masked_attention(q, k, v, mask, N, bq, bk, scale)
    for h in range(H):
        Ob, Lb = brute_attention(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), mask[h].tolist(), N, bq, bk, scale)
        np.testing.assert_allclose(O[0, h], Ob, atol=1e-12, rtol=0)
        np.testing.assert_array_equal(np.isneginf(L[0, h]), np.isneginf(Lb))
        fin = np.isfinite(Lb)
        np.testing.assert_allclose(L[0, h][fin], Lb[fin], atol=1e-12, rtol=0)


def test_zero_query_gives_mean_of_kept_values():
    # q = 0: every kept key scores 0, so O is the plain mean of the kept, real
    # values and LSE = log(#kept real keys).  An asymmetric mask catches a
    # swapped (query block, key block) index; a ragged N catches padding.
    H, N, Np, d, bq, bk = 1, 22, 24, 3, 8, 4
    q = np.zeros((1, H, Np, d))
    k = RNG.standard_normal((1, H, Np, d))
    v = RNG.standard_normal((1, H, Np, d))
    mask = np.zeros((H, 3, 6), np.uint8)
    mask[0, 0, [1, 5]] = 1
    mask[0, 1, [0]] = 1
    mask[0, 2, [2, 3, 5]] = 1
    O, L = oracle.masked_attention(q, k, v, mask, N, bq, bk, 1.0)
    for i in range(N):
        keys = [j for j in range(N) if mask[0, i // bq, j // bk]]
        np.testing.assert_allclose(O[0, 0, i], v[0, 0, keys].mean(axis=0), atol=1e-14)
        assert L[0, 0, i] == pytest.approx(math.log(len(keys)), abs=1e-14)


def test_block_diagonal_equals_independent_blocks():
    H, N, Np, d, blk = 2, 40, 40, 6, 8
    q, k, v = (RNG.standard_normal((1, H, Np, d)) for _ in range(3))
    mask = np.stack([np.eye(Np // blk, dtype=np.uint8)] * H)
    O, _ = oracle.masked_attention(q, k, v, mask, N, blk, blk, 0.5)
    for h in range(H):
        for b0 in range(0, N, blk):
            sl = slice(b0, b0 + blk)
            np.testing.assert_allclose(O[0, h, sl], sdpa64(q[0, h, sl], k[0, h, sl], v[0, h, sl], 0.5), atol=1e-12)


def test_constant_value_block_and_skipped_blocks_are_inert():
    H, N, Np, d, blk = 1, 32, 32, 4, 8
    q, k, v = (RNG.standard_normal((1, H, Np, d)) for _ in range(3))
    mask = np.zeros((H, 4, 4), np.uint8)
    mask[0, :, 2] = 1                       # one kept key block per row
    v2 = v.copy()
    v2[0, 0, 16:24] = np.array([1.5, -2.0, 0.25, 7.0])
    O, _ = oracle.masked_attention(q, k, v2, mask, N, blk, blk, 1.0)
    np.testing.assert_allclose(O[0, 0, :N], np.tile([1.5, -2.0, 0.25, 7.0], (N, 1)), atol=1e-13)
    # perturbing skipped keys/values changes nothing; perturbing kept ones does
    k3, v3 = k.copy(), v.copy()
    k3[0, 0, :16] += 5.0
    v3[0, 0, 24:] -= 3.0
    Oa, La = oracle.masked_attention(q, k, v, mask, N, blk, blk, 1.0)
    Ob, Lb = oracle.masked_attention(q, k3, v3, mask, N, blk, blk, 1.0)
    np.testing.assert_array_equal(Oa, Ob)
    np.testing.assert_array_equal(La, Lb)
    k4 = k.copy()
    k4[0, 0, 17] += 1.0
    Oc, _ = oracle.masked_attention(q, k4, v, mask, N, blk, blk, 1.0)
    assert np.abs(Oc - Oa).max() > 1e-6


def test_softmax_rows_sum_to_one():
    # the oracle's output with V = I (d = N) is the probability matrix itself
    H, N, blk = 1, 16, 4
    q = RNG.standard_normal((1, H, N, N))
    k = RNG.standard_normal((1, H, N, N))
    v = np.eye(N)[None, None]
    mask = (RNG.random((H, 4, 4)) < 0.6).astype(np.uint8)
    mask[0, np.arange(4), np.arange(4)] = 1
    P, _ = oracle.masked_attention(q, k, v, mask, N, blk, blk, 0.3)
    np.testing.assert_allclose(P[0, 0].sum(axis=1), 1.0, atol=1e-12)
    for i in range(N):
        for j in range(N):
            if not mask[0, i // blk, j // blk]:
                assert P[0, 0, i, j] == 0.0


# ----------------------------------------------------------------- O2 energy

def test_energy_rows_sum_to_one_and_uniform_closed_form():
    H, N, Np, d, blk = 2, 37, 40, 4, 8
    q = RNG.standard_normal((H, Np, d))
    k = RNG.standard_normal((H, Np, d))
    E = oracle.block_energy(q, k, N, blk, blk, 0.7)
    nq_real = math.ceil(N / blk)
    np.testing.assert_allclose(E[:, :nq_real].sum(axis=2), 1.0, atol=1e-12)
    # q = 0: uniform attention, E[qb, kb] = (#real keys in kb) / N
    E0 = oracle.block_energy(np.zeros_like(q), k, N, blk, blk, 0.7)
    counts = np.array([min(blk, max(0, N - kb * blk)) for kb in range(Np // blk)]) / N
    np.testing.assert_allclose(E0[:, :nq_real], np.broadcast_to(counts, E0[:, :nq_real].shape), atol=1e-14)


def test_energy_one_hot_closed_form():
    # q = k = c * I: s_ii = scale * c^2, s_ij = 0 (i != j), so
    # p_ii = e^a / (e^a + N - 1) and p_ij = 1 / (e^a + N - 1), a = scale * c^2.
    N, blk, c, scale = 12, 4, 2.0, 0.5
    q = (c * np.eye(N))[None]
    E = oracle.block_energy(q, q.copy(), N, blk, blk, scale)
    ea = math.exp(scale * c * c)
    z = ea + N - 1
    for qb in range(3):
        for kb in range(3):
            want = (ea + (blk - 1)) / z if qb == kb else blk / z
            assert E[0, qb, kb] == pytest.approx(want, abs=1e-14)


def test_energy_brute_force():
    N, blk, d = 10, 4, 3
    q = RNG.standard_normal((1, 12, d))
    k = RNG.standard_normal((1, 12, d))
    E = oracle.block_energy(q, k, N, blk, blk, 0.9)
    for qb in range(3):
        rows = [i for i in range(qb * blk, min(qb * blk + blk, N))]
        for kb in range(3):
            tot = 0.0
            for i in rows:
                s = [0.9 * math.fsum(q[0, i, t] * k[0, j, t] for t in range(d)) for j in range(N)]
                z = math.fsum(math.exp(x) for x in s)
                tot += math.fsum(math.exp(s[j]) / z for j in range(kb * blk, min(kb * blk + blk, N)))
            assert E[0, qb, kb] == pytest.approx(tot / len(rows), abs=1e-13)


def test_energy_non_square_blocks_brute_force_and_closed_form():
    # Table S6 key grids: key blocks of a size other than the query block's,
    # a ragged last key block, and a key grid of ceil(N / block_k) blocks
    # that ignores the query padding (N = 10, Np = 12, 3-key blocks -> 4).
    N, bq, bk, d, scale = 10, 4, 3, 3, 0.8
    q = RNG.standard_normal((1, 12, d))
    k = RNG.standard_normal((1, 12, d))
    E = oracle.block_energy(q, k, N, bq, bk, scale)
    assert E.shape == (1, 3, 4)
    for qb in range(3):
        rows = list(range(qb * bq, min(qb * bq + bq, N)))
        for kb in range(4):
            tot = 0.0
            for i in rows:
                s = [scale * math.fsum(q[0, i, t] * k[0, j, t] for t in range(d)) for j in range(N)]
                z = math.fsum(math.exp(x) for x in s)
                tot += math.fsum(math.exp(s[j]) / z for j in range(kb * bk, min(kb * bk + bk, N)))
            assert E[0, qb, kb] == pytest.approx(tot / len(rows), abs=1e-13)
    # q = 0: uniform attention, E[qb, kb] = (#real keys in kb) / N = 3, 3, 3, 1 tenths
    E0 = oracle.block_energy(np.zeros_like(q), k, N, bq, bk, scale)
    np.testing.assert_allclose(E0[0], np.broadcast_to([0.3, 0.3, 0.3, 0.1], (3, 4)), atol=1e-15)


# ----------------------------------------------------------------- O3 select

def test_topk_count_and_brute_force_order():
    assert oracle.topk_count(0.25, 256) == 64
    assert oracle.topk_count(0.2, 591) == 119
    assert oracle.topk_count(1e-9, 10) == 1
    assert oracle.topk_count(1.0, 10) == 10
    E = RNG.random((5, 7, 13))
    E[0, 0, 3] = E[0, 0, 9]                # a tie
    keep = oracle.select_topk(E, 0.3)
    k = math.ceil(0.3 * 13)
    assert np.all(keep.sum(axis=-1) == k)
    for idx in np.ndindex(5, 7):
        row = E[idx].tolist()
        want = sorted(range(13), key=lambda j: (-row[j], j))[:k]
        assert sorted(np.nonzero(keep[idx])[0].tolist()) == sorted(want)


def test_topk_ties_keep_smallest_indices():
    keep = oracle.select_topk(np.full((1, 10), 0.1), 0.35)
    assert keep[0].tolist() == [1, 1, 1, 1, 0, 0, 0, 0, 0, 0]


def test_energy_select_is_minimal_prefix_exact():
    # dyadic energies: every partial sum is exact, so Fractions decide the answer
    for trial in range(50):
        r = np.random.default_rng(trial)
        nkb = int(r.integers(1, 20))
        vals = r.integers(0, 64, nkb)
        E = (vals / 64.0)[None]
        eps = float(r.choice([0.0, 0.25, 0.5, 0.125, 0.9]))
        keep = oracle.select_energy(E, eps)[0]
        order = sorted(range(nkb), key=lambda j: (-vals[j], j))
        target = (1 - Fraction(eps)) * Fraction(int(vals.sum()), 64)
        run, want = Fraction(0), set()
        for j in order:
            want.add(j)
            run += Fraction(int(vals[j]), 64)
            if run >= target:
                break
        assert set(np.nonzero(keep)[0].tolist()) == want


# ----------------------------------------------------------------- O4 vote

def test_min_votes_for():
    assert oracle.min_votes_for(0.5, 8) == 4
    assert oracle.min_votes_for(0.3, 10) == 3
    assert oracle.min_votes_for(1.0, 7) == 7
    assert oracle.min_votes_for(0.0, 7) == 0
    assert oracle.min_votes_for(0.51, 8) == 5


def test_vote_invariants():
    I, H, nqb, nkb = 6, 3, 5, 9
    keeps = (RNG.random((I, H, nqb, nkb)) < 0.4).astype(np.uint8)
    keeps[:, 0, 0, 4] = 1                       # kept by every input
    keeps[:, 1, 2, :] = 0                       # never kept -> guard must fire
    keeps[0, 1, 2, 7] = 1                       # ... and pick the most-voted block
    E = RNG.random((I, H, nqb, nkb)).astype(np.float32)
    for mv in range(1, I + 1):
        mask, votes, esum = oracle.vote(keeps, mv, E)
        assert np.array_equal(votes, keeps.sum(axis=0))
        allkept = keeps.all(axis=0)
        assert np.all(mask[allkept] == 1)            # Figure 3(b): frequency 1 => computed
        assert np.all(mask.sum(axis=-1) >= 1)
        rowsempty = ~(votes >= mv).any(axis=-1)
        plain = (votes >= mv).astype(np.uint8)
        assert np.array_equal(mask[~rowsempty], plain[~rowsempty])
        assert np.all(mask[rowsempty].sum(axis=-1) == 1)
        assert mask[1, 2, 7] == 1 and mask[1, 2].sum() == 1
    union, _, _ = oracle.vote(keeps, 1, E)
    inter, _, _ = oracle.vote(keeps, I, E)
    nonempty_u = keeps.any(axis=0).any(axis=-1)
    assert np.array_equal(union[nonempty_u], keeps.any(axis=0).astype(np.uint8)[nonempty_u])
    nonempty_i = keeps.all(axis=0).any(axis=-1)
    assert np.array_equal(inter[nonempty_i], keeps.all(axis=0).astype(np.uint8)[nonempty_i])


def test_vote_guard_tie_break():
    keeps = np.zeros((2, 1, 1, 5), np.uint8)
    keeps[0, 0, 0, 1] = 1
    keeps[1, 0, 0, 3] = 1
    E = np.zeros((2, 1, 1, 5), np.float32)
    E[:, 0, 0, 3] = 0.25
    E[:, 0, 0, 1] = 0.25
    mask, _, _ = oracle.vote(keeps, 2, E)     # votes tie (1, 1); energy ties; smaller index wins
    assert mask[0, 0].tolist() == [0, 1, 0, 0, 0]
    E[1, 0, 0, 3] = 0.5
    mask, _, _ = oracle.vote(keeps, 2, E)     # larger energy sum wins
    assert mask[0, 0].tolist() == [0, 0, 0, 1, 0]


# ----------------------------------------------------------------- O5 compile

def test_compile_round_trip_and_counts():
    masks = (RNG.random((4, 11, 13)) < 0.3).astype(np.uint8)
    masks[1, 3] = 0
    for dedup in (True, False):
        bl = oracle.compile_blocklist(masks, dedup=dedup)
        assert np.array_equal(oracle.expand_blocklist(bl), masks)
        assert bl["nnz"] == int(masks.sum())
        rows = masks.reshape(-1, 13)
        for r in range(rows.shape[0]):
            cols = bl["csr_col"][bl["csr_row_ptr"][r]:bl["csr_row_ptr"][r + 1]]
            assert cols.tolist() == np.nonzero(rows[r])[0].tolist()
        assert bl["row_pat"][1 * 11 + 3] == 0 and bl["pat_ptr"][0] == bl["pat_ptr"][1] == 0
    bl = oracle.compile_blocklist(masks, dedup=False)
    assert bl["n_pat"] == 1 + int((masks.reshape(-1, 13).sum(axis=1) > 0).sum())


def test_compile_banded_closed_form():
    # |qb - kb| <= w on an n x n grid: rows are translates of w + 1 distinct
    # offset lists {0..L-1}, L = w+1 .. 2w+1 (top and bottom edge rows of equal
    # length coincide), so n_pat = w + 2 with the empty pattern.
    n, w = 20, 3
    m = np.zeros((1, n, n), np.uint8)
    for i in range(n):
        m[0, i, max(0, i - w):min(n, i + w + 1)] = 1
    bl = oracle.compile_blocklist(m)
    assert bl["n_pat"] == w + 2
    for p in range(1, w + 2):   # first occurrence order: row p-1 has length w + p
        lst = bl["pat_off"][bl["pat_ptr"][p]:bl["pat_ptr"][p + 1]]
        assert lst.tolist() == list(range(w + p))
    assert bl["row_pat"][n - 1] == 1 and bl["row_base"][n - 1] == n - 1 - w


def test_compile_empty_and_full():
    bl = oracle.compile_blocklist(np.zeros((2, 3, 4), np.uint8))
    assert bl["n_pat"] == 1 and bl["nnz"] == 0 and bl["nnz_pat"] == 0
    bl = oracle.compile_blocklist(np.ones((2, 3, 4), np.uint8))
    assert bl["n_pat"] == 2 and bl["nnz_pat"] == 4 and np.all(bl["row_pat"] == 1) and np.all(bl["row_base"] == 0)


# ---------------------------------------------------------------- O6 timestep sharing

def test_skipped_iou_hand_cases():
    # skipped sets {1, 2} and {2, 3}: intersection 1, union 3
    assert oracle.skipped_iou([1, 0, 0, 1], [1, 1, 0, 0]) == pytest.approx(1 / 3)
    assert oracle.skipped_iou([0, 1, 0], [0, 1, 0]) == 1.0
    assert oracle.skipped_iou([0, 1, 1], [1, 0, 1]) == 0.0           # disjoint skipped sets
    assert oracle.skipped_iou([1, 1], [1, 1]) == 1.0                 # nothing skipped: identical


def test_skipped_iou_matches_set_arithmetic():
    rng = np.random.default_rng(3)
    for _ in range(50):
        a = (rng.random(37) < 0.6).astype(np.uint8)
        b = (rng.random(37) < 0.6).astype(np.uint8)
        sa = {i for i in range(37) if a[i] == 0}
        sb = {i for i in range(37) if b[i] == 0}
        want = 1.0 if not (sa | sb) else len(sa & sb) / len(sa | sb)
        assert oracle.skipped_iou(a, b) == want


def _runs_masks():
    # one layer, one head, 4 timesteps: t0 == t1, t2 == t3, t1 and t2 far apart
    base = np.zeros((4, 4), np.uint8)
    m0 = base.copy(); m0[0, :] = 1
    m2 = base.copy(); m2[:, 3] = 1; m2[1, :] = 1
    return np.stack([m0, m0, m2, m2])[None, :, None]


def test_timestep_clusters_hand_case_and_extremes():
    masks = _runs_masks()
    assert oracle.timestep_clusters(masks, 0.9).tolist() == [[0, 0, 1, 1]]
    assert oracle.timestep_clusters(masks, 0.0).tolist() == [[0, 0, 0, 0]]
    assert oracle.timestep_clusters(masks, 1.01).tolist() == [[0, 1, 2, 3]]


def test_timestep_clusters_are_pairwise_and_greedy():
    rng = np.random.default_rng(11)
    L, T, H = 3, 7, 2
    base = rng.random((L, 1, H, 6, 6)) < 0.5
    flips = rng.random((L, T, H, 6, 6)) < rng.choice([0.02, 0.1, 0.4], size=(L, T, 1, 1, 1))
    masks = (base ^ np.cumsum(flips, axis=1).astype(bool)).astype(np.uint8)
    for tau in (0.3, 0.6, 0.9):
        cl = oracle.timestep_clusters(masks, tau)
        for l in range(L):
            ids = cl[l].tolist()
            assert ids[0] == 0 and all(b - a in (0, 1) for a, b in zip(ids, ids[1:]))   # consecutive runs
            for c in set(ids):
                mem = [t for t in range(T) if ids[t] == c]
                for t1 in mem:                                                          # pair-wise >= tau
                    for t2 in mem:
                        if t1 != t2:
                            sim = np.mean([oracle.skipped_iou(masks[l, t1, h], masks[l, t2, h]) for h in range(H)])
                            assert sim >= tau
            for t in range(1, T):                                                       # greedy: a new run
                if ids[t] != ids[t - 1]:                                                # had a reason to start
                    prev = [s for s in range(t) if ids[s] == ids[t - 1]]
                    sims = [np.mean([oracle.skipped_iou(masks[l, t, h], masks[l, s, h]) for h in range(H)])
                            for s in prev]
                    assert min(sims) < tau


def test_share_masks_union_and_offsets():
    masks = _runs_masks()
    cl = oracle.timestep_clusters(masks, 0.9)
    shared, off = oracle.share_masks(masks, cl)
    assert shared.shape == (2, 1, 4, 4)
    assert off.tolist() == [[0, 0, 1, 1]]
    for t in range(4):
        got = shared[off[0, t]]
        assert np.all(got >= masks[0, t])                 # nothing a member keeps is skipped
    singleton = oracle.share_masks(masks, np.array([[0, 1, 2, 3]]))[0]
    assert np.array_equal(singleton[:, 0], masks[0, :, 0])


# ---------------------------------------------------------------- O7 interval skip lists

def test_interval_counts_hand_and_brute_force():
    rows = np.array([[[1, 1, 0, 1, 0, 0, 1], [0] * 7, [1] * 7, [1, 0, 1, 0, 1, 0, 1]]], np.uint8)
    assert oracle.interval_counts(rows).tolist() == [[3, 0, 1, 4]]
    rng = np.random.default_rng(2)
    m = (rng.random((3, 5, 41)) < 0.5).astype(np.uint8)
    want = [[sum(1 for i in range(41) if m[a, b, i] and (i == 0 or not m[a, b, i - 1])) for b in range(5)]
            for a in range(3)]
    assert oracle.interval_counts(m).tolist() == want


def test_merge_row_hand_cases():
    assert oracle.merge_row([1, 0, 1, 0, 0, 1], 2).tolist() == [1, 1, 1, 0, 0, 1]     # smallest gap first
    assert oracle.merge_row([1, 0, 1, 0, 0, 1], 1).tolist() == [1] * 6
    assert oracle.merge_row([0, 1, 0, 0, 1, 0, 0, 1, 0], 2).tolist() == [0, 1, 1, 1, 1, 0, 0, 1, 0]  # tie: leftmost
    assert oracle.merge_row([0, 0, 0], 1).tolist() == [0, 0, 0]
    assert oracle.merge_row([1, 0, 1], 5).tolist() == [1, 0, 1]


def test_merge_row_invariants():
    rng = np.random.default_rng(7)
    for _ in range(200):
        n = int(rng.integers(1, 60))
        row = (rng.random(n) < rng.random()).astype(np.uint8)
        width = int(rng.integers(1, 8))
        out = oracle.merge_row(row, width)
        cnt = int(oracle.interval_counts(row[None, None])[0, 0])
        cnt_out = int(oracle.interval_counts(out[None, None])[0, 0])
        assert np.all(out >= row)
        assert cnt_out == min(cnt, width) if cnt else cnt_out == 0
        kept = np.nonzero(row)[0]
        if kept.size:
            assert not out[:kept[0]].any() and not out[kept[-1] + 1:].any()
        # the gaps filled are the smallest ones
        gaps = []
        i = 0
        while i < n:
            if row[i] == 0 and 0 < i and kept.size and kept[0] < i < kept[-1]:
                j = i
                while row[j] == 0:
                    j += 1
                gaps.append((j - i, bool(out[i])))
                i = j
            else:
                i += 1
        filled = [g for g, f in gaps if f]
        unfilled = [g for g, f in gaps if not f]
        assert len(filled) == max(0, cnt - width)
        if filled and unfilled:
            assert max(filled) <= min(unfilled)


def test_nearest_rank_and_skiplist_bytes():
    assert oracle.nearest_rank([4, 1, 3, 2], 50) == 2
    assert oracle.nearest_rank([4, 1, 3, 2], 100) == 4
    assert oracle.nearest_rank(list(range(1, 21)), 95) == 19
    counts = np.array([[1, 3], [2, 2]])        # two layers of one map with two rows each
    b = oracle.skiplist_bytes(counts, 1, 5, pct=50)
    assert b == {"full": 2 * 2 * 3 * 8, "trimmed": 2 * 3 * 8 + 2 * 2 * 8, "merged": 2 * 1 * 8 + 2 * 2 * 8}


# ---------------------------------------------------------------- O8 spatial repetition

def test_anchor_rows_match_table_s4_row_sparsity_and_nearest():
    import json
    from pathlib import Path
    g = json.loads((Path(__file__).parent / "golden" / "geometry.json").read_text())["table_s4_anchor_rows"]
    for k, pct in zip(g["k"], g["sparsity_pct"]):
        anchors, nearest = oracle.anchor_rows(30, k)
        assert len(set(anchors)) == k
        assert round(100.0 * (1 - len(set(anchors)) / 30), 1) == pct
        for r in range(30):                        # nearest by brute force, ties to the lower anchor
            dists = sorted((abs(a - r), a) for a in anchors)
            assert nearest[r] == dists[0][1]
    assert oracle.anchor_rows(30, 4)[0] == [3, 11, 18, 26]
    assert oracle.anchor_rows(30, 4)[1][7] == 3     # |7-3| == |11-7|: the lower anchor
    assert oracle.anchor_rows(12, 12) == (list(range(12)), list(range(12)))


def test_anchor_attention_against_sdpa():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(21)
    frames, rows, cols, d = 2, 6, 5, 16
    N = frames * rows * cols
    Np = N + 4
    q, k, v = (rng.standard_normal((1, 2, Np, d)) for _ in range(3))
    scale = 0.3
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[:, :, :N]), torch.from_numpy(k[:, :, :N]), torch.from_numpy(v[:, :, :N]),
        scale=scale).numpy()
    full = oracle.anchor_attention(q, k, v, N, frames, rows, cols, rows, scale)   # every row an anchor
    assert np.allclose(full[:, :, :N], ref, atol=1e-12) and not full[:, :, N:].any()
    o = oracle.anchor_attention(q, k, v, N, frames, rows, cols, 2, scale)
    anchors, nearest = oracle.anchor_rows(rows, 2)
    for f in range(frames):
        for r in range(rows):
            for c in range(cols):
                t = f * rows * cols + r * cols + c
                ta = f * rows * cols + nearest[r] * cols + c
                assert np.allclose(o[:, :, t], ref[:, :, ta], atol=1e-12)
    # the per-token form: the same values for a token subset, zeros past N
    toks = [0, 7, 31, N - 1, N + 2]
    for h in range(2):
        sub = oracle.anchor_attention_tokens(q, k, v, N, frames, rows, cols, 2, scale, 0, h, toks)
        want = [ref[0, h, f * rows * cols + nearest[(t % (rows * cols)) // cols] * cols + t % cols]
                if t < N else np.zeros(d) for t in toks for f in [t // (rows * cols)]]
        assert np.allclose(sub, np.stack(want), atol=1e-12)


def test_block_energy_row_is_a_row_of_block_energy():
    rng = np.random.default_rng(5)
    H, N, Np, d = 2, 300, 384, 16
    q = rng.standard_normal((H, Np, d))
    k = rng.standard_normal((H, Np, d))
    E = oracle.block_energy(q, k, N, 128, 64, 0.25)
    for h, qb in ((0, 0), (1, 2), (1, 1)):
        assert np.array_equal(oracle.block_energy_row(q, k, N, 128, 64, 0.25, h, qb), E[h, qb])


def _sim_video(frames, rows, cols, text, d, rng, same_rows=False):
    N = frames * rows * cols + text
    q = rng.standard_normal((2, N + 3, d))
    if same_rows:   # every spatial row of a frame repeats the first one (per frame and column)
        for f in range(frames):
            for r in range(1, rows):
                q[:, (f * rows + r) * cols:(f * rows + r + 1) * cols] = q[:, f * rows * cols:(f * rows + 1) * cols]
    k = rng.standard_normal((2, N + 3, d))
    return q, k, N


def test_spatial_similarity_closed_forms():
    rng = np.random.default_rng(31)
    # rows that repeat within each frame (and differ across frames and columns): score 1
    q, k, N = _sim_video(3, 4, 5, 7, 6, rng, same_rows=True)
    assert np.allclose(oracle.spatial_similarity(q, k, N, 3, 4, 5, 0.7), 1.0, atol=1e-12)
    # one-hot attention on distinct keys: neighbouring rows share nothing, score 0
    frames, rows, cols = 2, 3, 4
    n = frames * rows * cols
    e = np.eye(n)[None].repeat(2, axis=0) * 40.0
    assert np.allclose(oracle.spatial_similarity(e, e, n, frames, rows, cols, 1.0), 0.0, atol=1e-12)


def test_spatial_similarity_brute_force():
    rng = np.random.default_rng(32)
    frames, rows, cols, text, d, scale = 2, 3, 2, 2, 4, 0.6
    q, k, N = _sim_video(frames, rows, cols, text, d, rng)
    got = oracle.spatial_similarity(q, k, N, frames, rows, cols, scale)
    for h in range(2):
        def prow(t):
            s = [scale * sum(q[h, t, x] * k[h, j, x] for x in range(d)) for j in range(N)]
            m = max(s)
            e = [math.exp(v - m) for v in s]
            z = math.fsum(e)
            return [v / z for v in e]
        cos = []
        for f in range(frames):
            for r in range(rows - 1):
                for c in range(cols):
                    a = prow((f * rows + r) * cols + c)
                    b = prow((f * rows + r + 1) * cols + c)
                    num = math.fsum(x * y for x, y in zip(a, b))
                    den = math.sqrt(math.fsum(x * x for x in a) * math.fsum(y * y for y in b))
                    cos.append(num / den)
        assert abs(got[h] - math.fsum(cos) / len(cos)) < 1e-12


def test_repetition_flags_hand_case():
    scores = np.array([[1.0, 0.5, 0.75], [0.5, 0.5, 1.0]], np.float32)
    mean, flags = oracle.repetition_flags(scores, 0.75)
    assert mean.tolist() == [0.75, 0.5, 0.875] and flags.tolist() == [1, 0, 1]
