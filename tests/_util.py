"""Helpers shared by the GPU parity tests (no method arithmetic here)."""

import numpy as np
import torch

from block_sparse_attention_cross_b200 import synthetic as syn

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_MAX_ABS = 1e-5


def bf16_pair(x_f32):
    """(exact float64 values for the oracle, bf16 CUDA tensor with the same values)."""
    bits = syn.f32_to_bf16_bits(x_f32)
    exact = syn.bf16_bits_to_f32(bits).astype(np.float64)
    dev = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return exact, dev


def fp32_pair(x_f32):
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    return x.astype(np.float64), torch.from_numpy(x).cuda()


def to_np64(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(got, want, max_abs, mean_abs=None, what="O"):
    err = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    mx = float(err.max()) if err.size else 0.0
    mn = float(err.mean()) if err.size else 0.0
    assert mx <= max_abs, f"{what}: max abs error {mx:.3e} > {max_abs:.1e} (mean {mn:.3e})"
    if mean_abs is not None:
        assert mn <= mean_abs, f"{what}: mean abs error {mn:.3e} > {mean_abs:.1e}"
    return mx, mn


def assert_lse(got, want, tol):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    ninf = np.isneginf(want)
    assert np.array_equal(np.isneginf(got), ninf), "LSE -inf pattern differs"
    if (~ninf).any():
        assert_close(got[~ninf], want[~ninf], tol, what="LSE")
