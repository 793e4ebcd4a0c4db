"""calibatt_block_energy_noalloc: block energies without any device allocation.

For callers that only hold their input and output buffers (a plugin whose
host engine gives it no workspace, or a service that reserved the GPU's
memory for its own pool and allows no allocation afterwards), the library
keeps the per-row scratch of the energy computation in a fixed array of its
own.  This checks, through the C ABI, that two calls in a row give exactly
the workspace-taking entry point's result (the same kernels run on the same
inputs, so the comparison is bit for bit), that a call with padded rows
(N < Np) made right after a call that filled every scratch row is not
affected by what that call left behind, and that a call too large for the
fixed array is refused before anything launches.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import _lib
from block_sparse_attention_cross_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

def _inputs(d, dtype, block, H=2, grid=syn.VideoGrid(2, 30, 52), seed=31):
    w = syn.Workload("noalloc", 1, H, grid, d, "bf16", block, 0.25,
                     {"base": seed, "noise_q": seed + 1, "noise_k": seed + 2, "v": seed + 3})
    q, k = syn.video_qkv(w, with_v=False)
    tdt = torch.bfloat16 if dtype == _lib.BF16 else torch.float32
    return w, torch.from_numpy(q[0]).cuda().to(tdt), torch.from_numpy(k[0]).cuda().to(tdt)


def _call_noalloc(lib, q, k, N, block, dtype, E, status):
    H, Np, d = q.shape
    return lib.calibatt_block_energy_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), H, N, Np, d, dtype, block, block,
        cba.default_scale(d), ctypes.c_void_p(E.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,d,block", [(_lib.BF16, 128, 128), (_lib.FP32, 64, 64)])
def test_noalloc_matches_workspace_entry_point_twice(dtype, d, block):
    lib = _lib.load()
    w, q, k = _inputs(d, dtype, block)
    assert w.N < w.Np
    ref = cba.block_energy(q, k, w.N, block, block)       # the existing entry point (caller workspace)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        E = torch.full_like(ref, float("nan"))
        rc = _call_noalloc(lib, q, k, w.N, block, dtype, E, status)
        assert rc == _lib.OK, lib.calibatt_last_error().decode()
        torch.cuda.synchronize()
        assert status.item() == 0
        assert torch.equal(E, ref)
    # a different input in between must not leave state behind
    w2, q2, k2 = _inputs(d, dtype, block, seed=77)
    ref2 = cba.block_energy(q2, k2, w2.N, block, block)
    E2 = torch.empty_like(ref2)
    assert _call_noalloc(lib, q2, k2, w2.N, block, dtype, E2, status) == _lib.OK
    torch.cuda.synchronize()
    assert torch.equal(E2, ref2)


@pytest.mark.parametrize("dtype,d,block", [(_lib.BF16, 128, 128), (_lib.FP32, 64, 64)])
def test_noalloc_padded_rows_after_a_full_call(dtype, d, block):
    # First a call with no padding (N = Np: every scratch row written with a
    # real log-sum-exp), then one on other inputs of the same Np with the last
    # five rows as padding: those rows' scratch entries still hold the first
    # call's values and must not reach the result.
    lib = _lib.load()
    w, q, k = _inputs(d, dtype, block, grid=syn.VideoGrid(2, 32, 50), seed=41)   # 3200 tokens, no padding
    assert w.N == w.Np
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    E = torch.empty((w.H, w.Np // block, w.Np // block), device="cuda", dtype=torch.float32)
    assert _call_noalloc(lib, q, k, w.N, block, dtype, E, status) == _lib.OK
    assert torch.equal(E, cba.block_energy(q, k, w.N, block, block))
    _, q2, k2 = _inputs(d, dtype, block, grid=syn.VideoGrid(2, 32, 50), seed=53)
    n2 = w.Np - 5
    ref2 = cba.block_energy(q2, k2, n2, block, block)
    E2 = torch.full_like(ref2, float("nan"))
    assert _call_noalloc(lib, q2, k2, n2, block, dtype, E2, status) == _lib.OK, lib.calibatt_last_error().decode()
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(E2, ref2)


def test_noalloc_rejects_calls_beyond_the_fixed_scratch():
    lib = _lib.load()
    H, Np, d = 129, 32768, 128                 # H * Np = 4 227 072 > 4 194 304 rows
    fake = ctypes.c_void_p(0x10000)
    rc = lib.calibatt_block_energy_noalloc(fake, fake, H, Np, Np, d, _lib.BF16, 128, 128, 0.088, fake, None, None)
    assert rc == _lib.E_WORKSPACE
    assert "exceeds the built-in scratch" in lib.calibatt_last_error().decode()
