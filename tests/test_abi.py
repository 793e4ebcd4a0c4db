"""The C-ABI library loads, exports every function include/calibatt.h declares,
and rejects bad arguments with status codes before touching the GPU.

These run without a GPU: every call below fails validation on the host, so
no CUDA call is made.
"""

import ctypes
import re
from pathlib import Path

import pytest

from block_sparse_attention_cross_b200 import _lib

HEADER = Path(__file__).resolve().parent.parent / "include" / "calibatt.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = set(re.findall(r"\b(calibatt_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_header_compiles_as_c_and_links(lib, tmp_path):
    # tests/c/abi_host.c: the header as C99 with strict warnings, linked
    # against the library, host-only calls answered from C
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    pkg = Path(_lib.LIB_PATH).parent
    exe = tmp_path / "abi_host"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", f"-I{HEADER.parent}",
                    str(Path(__file__).resolve().parent / "c" / "abi_host.c"), f"-L{pkg}", "-lcalibatt",
                    f"-Wl,-rpath,{pkg}", "-o", str(exe)], check=True, timeout=120)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout


def test_header_and_binding_agree():
    names = declared_functions()
    assert len(names) >= 14
    assert set(names) == set(_lib.EXPORTS), set(names) ^ set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_counters(lib):
    assert lib.calibatt_version() == 10000
    assert lib.calibatt_launch_count() == 0 or lib.calibatt_launch_count() > 0
    old = lib.calibatt_get_spin_limit_ns()
    assert old > 0
    lib.calibatt_set_spin_limit_ns(12345)
    assert lib.calibatt_get_spin_limit_ns() == 12345
    lib.calibatt_set_spin_limit_ns(old)


def _err(lib):
    return lib.calibatt_last_error().decode()


def test_fwd_rejects_null_and_bad_sizes(lib):
    bl = _lib.Blocklist()
    rc = lib.calibatt_sparse_attn_fwd(None, None, None, None, None, 1, 1, 128, 128, 128, _lib.BF16, 0.1,
                                      ctypes.byref(bl), 0, None, None)
    assert rc == _lib.E_INVALID and "non-NULL" in _err(lib)
    fake = ctypes.c_void_p(0x10000)
    rc = lib.calibatt_sparse_attn_fwd(fake, fake, fake, fake, None, 1, 1, 200, 128, 128, _lib.BF16, 0.1,
                                      ctypes.byref(bl), 0, None, None)
    assert rc == _lib.E_INVALID                       # Np < N
    rc = lib.calibatt_sparse_attn_fwd(fake, fake, fake, fake, None, 1, 1, 128, 128, 128, _lib.BF16, -1.0,
                                      ctypes.byref(bl), 0, None, None)
    assert rc == _lib.E_INVALID and "scale" in _err(lib)
    rc = lib.calibatt_sparse_attn_fwd(ctypes.c_void_p(0x10001), fake, fake, fake, None, 1, 1, 128, 128, 128,
                                      _lib.BF16, 0.1, ctypes.byref(bl), 0, None, None)
    assert rc == _lib.E_INVALID and "aligned" in _err(lib)
    rc = lib.calibatt_sparse_attn_fwd(fake, fake, fake, fake, None, 1, 1, 128, 128, 128, _lib.BF16, 0.1,
                                      None, 0, None, None)
    assert rc == _lib.E_INVALID and "block list" in _err(lib)


def _blocklist(n_maps, nq, nk, bq, bk):
    bl = _lib.Blocklist()
    bl.n_maps, bl.n_q_blocks, bl.n_k_blocks, bl.block_q, bl.block_k = n_maps, nq, nk, bq, bk
    bl.row_base = bl.row_pat = bl.pat_ptr = bl.pat_off = 0x20000
    bl.n_pat, bl.nnz_pat, bl.nnz = 1, 0, 0
    return bl


def test_fwd_rejects_mismatched_blocklist_and_unsupported(lib):
    fake = ctypes.c_void_p(0x10000)
    bl = _blocklist(2, 8, 8, 128, 128)
    args = lambda B, H, N, Np, d, dt, mo: (fake, fake, fake, fake, None, B, H, N, Np, d, dt, 0.1,
                                           ctypes.byref(bl), mo, None, None)
    assert lib.calibatt_sparse_attn_fwd(*args(1, 2, 1000, 1024, 128, _lib.BF16, 1)) == _lib.E_INVALID  # map range
    assert "map_offset" in _err(lib)
    assert lib.calibatt_sparse_attn_fwd(*args(1, 2, 1000, 896, 128, _lib.BF16, 0)) == _lib.E_INVALID   # grid
    assert lib.calibatt_sparse_attn_fwd(*args(1, 2, 1000, 1024, 96, _lib.BF16, 0)) == _lib.E_UNSUPPORTED
    assert lib.calibatt_sparse_attn_fwd(*args(1, 2, 1000, 1024, 128, 7, 0)) == _lib.E_UNSUPPORTED
    bl64 = _blocklist(2, 16, 16, 64, 64)
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, fake, None, 1, 2, 1024, 1024, 128, _lib.BF16, 0.1,
                                        ctypes.byref(bl64), 0, None, None) == _lib.E_UNSUPPORTED
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, fake, None, 1, 2, 1024, 1024, 32, _lib.FP32, 0.1,
                                        ctypes.byref(bl64), 0, None, None) == _lib.E_UNSUPPORTED
    # padding of a whole block is rejected
    assert lib.calibatt_sparse_attn_fwd(*args(1, 2, 896, 1024, 128, _lib.BF16, 0)) == _lib.E_INVALID


def test_streamed_fwd_checks_everything_before_enqueueing(lib):
    # Every rejection below happens on the host before any stream, event or
    # copy is created, so no CUDA call is made.
    fake = ctypes.c_void_p(0x10000)
    host = ctypes.c_void_p(0x30000)
    bl = _blocklist(2, 8, 8, 128, 128)

    def call(qh=host, oh=host, lh=None, qd=fake, ld=None, B=1, H=2, N=1000, Np=1024, d=128, dt=_lib.BF16, mo=0,
             hpc=1, blp=ctypes.byref(bl)):
        return lib.calibatt_sparse_attn_fwd_streamed(qh, host, host, oh, lh, qd, fake, fake, fake, ld, B, H, N, Np,
                                                     d, dt, 0.1, blp, mo, hpc, None, None)

    assert call(qh=None) == _lib.E_INVALID and "host" in _err(lib)
    assert call(oh=None) == _lib.E_INVALID
    assert call(qd=None) == _lib.E_INVALID and "dev" in _err(lib)
    assert call(lh=host) == _lib.E_INVALID and "lse" in _err(lib)        # lse_host without lse_dev
    assert call(ld=fake) == _lib.E_INVALID and "lse" in _err(lib)        # lse_dev without lse_host
    assert call(hpc=0) == _lib.E_INVALID and "heads_per_chunk" in _err(lib)
    assert call(mo=1) == _lib.E_INVALID and "map_offset" in _err(lib)
    assert call(d=96) == _lib.E_UNSUPPORTED
    assert call(dt=7) == _lib.E_UNSUPPORTED
    assert call(qd=ctypes.c_void_p(0x10008)) == _lib.E_INVALID and "aligned" in _err(lib)
    assert call(blp=None) == _lib.E_INVALID and "block list" in _err(lib)


def test_workspace_queries(lib):
    n = ctypes.c_size_t(0)
    assert lib.calibatt_calibrate_workspace_size(40, 32760, 32768, 128, 128, 128, ctypes.byref(n)) == _lib.OK
    assert n.value >= 40 * 32768 * 4 + 40 * 256 * 256 * 4
    assert lib.calibatt_calibrate_workspace_size(40, 32760, 32760, 128, 128, 128, ctypes.byref(n)) == _lib.E_INVALID
    # key blocks of 80 over 32 760 real keys: ceil(32760 / 80) = 410 blocks per row
    assert lib.calibatt_calibrate_workspace_size(40, 32760, 32768, 128, 128, 80, ctypes.byref(n)) == _lib.OK
    assert n.value >= 40 * 32768 * 4 + 40 * 256 * 410 * 4
    assert lib.calibatt_compile_workspace_size(4800, 256, 256, ctypes.byref(n)) == _lib.OK
    assert n.value > 4800 * 256 * 8
    assert lib.calibatt_compile_workspace_size(0, 256, 256, ctypes.byref(n)) == _lib.E_INVALID


def test_calibration_and_compile_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    assert lib.calibatt_block_energy(fake, fake, 2, 1000, 1024, 128, _lib.BF16, 64, 64, 0.1, fake, fake, 1 << 30,
                                     None, None) == _lib.E_UNSUPPORTED
    assert lib.calibatt_block_energy(fake, fake, 2, 1000, 1024, 128, _lib.BF16, 128, 128, 0.1, fake, fake, 16,
                                     None, None) == _lib.E_WORKSPACE
    # Table S6 key blocks pass validation (then fail on the workspace); others are unsupported
    for bk in (64, 80, 96, 144):
        assert lib.calibatt_block_energy(fake, fake, 2, 1000, 1024, 128, _lib.BF16, 128, bk, 0.1, fake, fake, 16,
                                         None, None) == _lib.E_WORKSPACE
    assert lib.calibatt_block_energy(fake, fake, 2, 1000, 1024, 128, _lib.BF16, 128, 112, 0.1, fake, fake, 1 << 30,
                                     None, None) == _lib.E_UNSUPPORTED
    # 2 048 query tiles of 128 rows with 64-key blocks: 4 096 key blocks per row, above the limit
    assert lib.calibatt_block_energy(fake, fake, 1, 262144, 262144, 64, _lib.BF16, 128, 64, 0.1, fake, fake,
                                     1 << 30, None, None) == _lib.E_UNSUPPORTED
    assert lib.calibatt_select_vote(fake, 2, 8, 8, 5, 0.1, fake, fake, None) == _lib.E_INVALID
    assert lib.calibatt_select_vote(fake, 2, 8, 8, _lib.SELECT_TOPK, 0.0, fake, fake, None) == _lib.E_INVALID
    assert lib.calibatt_select_vote(fake, 2, 8, 8, _lib.SELECT_ENERGY, 1.0, fake, fake, None) == _lib.E_INVALID
    assert lib.calibatt_finalize_mask(fake, fake, 2, 8, 8, -1, fake, None) == _lib.E_INVALID
    # H * nqb rows at 2^31 would overflow the row index: refused before any launch
    assert lib.calibatt_select_vote(fake, 65536, 32768, 8, _lib.SELECT_TOPK, 0.25, fake, fake, None) == \
        _lib.E_UNSUPPORTED
    assert lib.calibatt_finalize_mask(fake, fake, 65536, 32768, 8, 1, fake, None) == _lib.E_UNSUPPORTED
    nnz, npat, nnzp = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    assert lib.calibatt_compile_size(fake, 1, 8, 40000, 1, ctypes.byref(nnz), ctypes.byref(npat), ctypes.byref(nnzp),
                                     fake, 1 << 20, None) == _lib.E_UNSUPPORTED
    assert lib.calibatt_compile_size(fake, 1, 8, 8, 9, ctypes.byref(nnz), ctypes.byref(npat), ctypes.byref(nnzp),
                                     fake, 1 << 20, None) == _lib.E_INVALID
    assert lib.calibatt_compile(fake, 1, 8, 8, 1, 128, 128, None, fake, 1 << 20, None) == _lib.E_INVALID
    assert lib.calibatt_selftest_wait_timeout(0, fake, None) == _lib.E_INVALID
    assert lib.calibatt_selftest_wait_timeout(1000, None, None) == _lib.E_INVALID


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    import block_sparse_attention_cross_b200 as cba
    x = torch.zeros(1, 1, 128, 64)
    with pytest.raises(ValueError):
        cba.sparse_attn_fwd(x, x, x, None, 128)


def test_timestep_sharing_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    run = (ctypes.c_int32 * 8)()
    n = ctypes.c_int32(0)
    size = ctypes.c_size_t(0)
    assert lib.calibatt_timestep_clusters_workspace_size(2, 4, 3, ctypes.byref(size)) == _lib.OK
    assert size.value == 2 * 2 * 3 * 4 * 4 * 8
    assert lib.calibatt_timestep_clusters(None, 2, 4, 3, 8, 8, 0.5, run, ctypes.byref(n), fake, size.value,
                                          None) == _lib.E_INVALID
    assert lib.calibatt_timestep_clusters(fake, 2, 2000, 3, 8, 8, 0.5, run, ctypes.byref(n), fake, 1 << 30,
                                          None) == _lib.E_UNSUPPORTED
    assert lib.calibatt_timestep_clusters(fake, 2, 4, 3, 8, 8, 0.5, run, ctypes.byref(n), fake, 16,
                                          None) == _lib.E_WORKSPACE
    assert lib.calibatt_timestep_clusters(fake, 2, 4, 3, 8, 8, float("nan"), run, ctypes.byref(n), fake,
                                          size.value, None) == _lib.E_INVALID
    assert lib.calibatt_share_masks(fake, 2, 4, 3, 8, 8, fake, 0, fake, None) == _lib.E_INVALID
    assert lib.calibatt_share_masks(fake, 2, 4, 3, 8, 8, fake, 9, fake, None) == _lib.E_INVALID


def test_documented_errors_of_the_auxiliary_calls(lib):
    # every case is refused on the host, before any launch
    fake = ctypes.c_void_p(0x10000)
    # one block per (run, head): n_runs * H above 65535 is unsupported
    assert lib.calibatt_share_masks(fake, 1024, 64, 2, 8, 8, fake, 40000, fake, None) == _lib.E_UNSUPPORTED
    # L * T above 2^20
    run = (ctypes.c_int32 * 1)()
    n = ctypes.c_int32(0)
    assert lib.calibatt_timestep_clusters(fake, 2048, 1024, 1, 8, 8, 0.5, run, ctypes.byref(n), fake, 1 << 30,
                                          None) == _lib.E_UNSUPPORTED
    bl = _blocklist(4, 8, 8, 128, 128)
    kept = ctypes.c_int64(0)
    assert lib.calibatt_blocklist_kept(None, 0, 1, ctypes.byref(kept), fake, 8, None) == _lib.E_INVALID
    assert lib.calibatt_blocklist_kept(ctypes.byref(bl), 3, 2, ctypes.byref(kept), fake, 8, None) == _lib.E_INVALID
    assert lib.calibatt_blocklist_kept(ctypes.byref(bl), -1, 2, ctypes.byref(kept), fake, 8, None) == _lib.E_INVALID
    assert lib.calibatt_blocklist_kept(ctypes.byref(bl), 0, 2, ctypes.byref(kept), fake, 4, None) == \
        _lib.E_WORKSPACE
    assert lib.calibatt_blocklist_kept(ctypes.byref(bl), 0, 2, ctypes.byref(kept), ctypes.c_void_p(0x10004), 8,
                                       None) == _lib.E_INVALID
    csr, pool = ctypes.c_int64(0), ctypes.c_int64(0)
    assert lib.calibatt_blocklist_bytes(2, 8, 10, 0, 4, ctypes.byref(csr), ctypes.byref(pool)) == _lib.E_INVALID
    assert lib.calibatt_blocklist_bytes(2, 8, -1, 3, 4, ctypes.byref(csr), ctypes.byref(pool)) == _lib.E_INVALID
    # the sizes themselves: int64 row pointers + int16 columns; int32 base and pattern id per row, int32 pattern
    # pointers, int16 offsets
    assert lib.calibatt_blocklist_bytes(2, 8, 10, 3, 4, ctypes.byref(csr), ctypes.byref(pool)) == _lib.OK
    assert (csr.value, pool.value) == (17 * 8 + 10 * 2, 16 * 8 + 4 * 4 + 4 * 2)
    assert lib.calibatt_selftest_wait_timeout(10_000_000_001, fake, None) == _lib.E_INVALID
    assert lib.calibatt_merge_intervals(fake, 2, -1, 8, fake, fake, None) == _lib.E_INVALID
    assert lib.calibatt_gather_rows(fake, fake, fake, 0, 4, 4, 256, None) == _lib.E_INVALID


def test_skiplist_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    assert lib.calibatt_interval_counts(None, 2, 8, 8, fake, None) == _lib.E_INVALID
    assert lib.calibatt_interval_counts(fake, 0, 8, 8, fake, None) == _lib.E_INVALID
    assert lib.calibatt_merge_intervals(fake, 2, 8, 8, None, fake, None) == _lib.E_INVALID
    assert lib.calibatt_merge_intervals(fake, 2, 8, 4096, fake, fake, None) == _lib.E_UNSUPPORTED


def test_gathered_query_forward_and_gather_validation(lib):
    fake = ctypes.c_void_p(0x10000)
    bl = _blocklist(2, 2, 8, 128, 128)
    # fp32 has no separate query / key lengths
    assert lib.calibatt_sparse_attn_fwd_qk(fake, fake, fake, fake, None, 1, 2, 200, 256, 1000, 1024, 128, _lib.FP32,
                                           0.1, ctypes.byref(bl), 0, None, None) == _lib.E_UNSUPPORTED
    # query grid must match Npq / 128
    assert lib.calibatt_sparse_attn_fwd_qk(fake, fake, fake, fake, None, 1, 2, 300, 384, 1000, 1024, 128, _lib.BF16,
                                           0.1, ctypes.byref(bl), 0, None, None) == _lib.E_INVALID
    # a whole padded query block is rejected
    assert lib.calibatt_sparse_attn_fwd_qk(fake, fake, fake, fake, None, 1, 2, 100, 256, 1000, 1024, 128, _lib.BF16,
                                           0.1, ctypes.byref(bl), 0, None, None) == _lib.E_INVALID
    assert lib.calibatt_gather_rows(None, fake, fake, 1, 4, 4, 256, None) == _lib.E_INVALID
    assert lib.calibatt_gather_rows(fake, fake, fake, 1, 4, 4, 200, None) == _lib.E_INVALID     # not a multiple of 16
    assert lib.calibatt_gather_rows(ctypes.c_void_p(0x10008), fake, fake, 1, 4, 4, 256, None) == _lib.E_INVALID


def test_integer_parameters_match_the_oracle(lib):
    # calibatt_min_votes / calibatt_topk_count are host arithmetic in the
    # library: the same integers as the oracle's definitions over a grid.
    import oracle
    import block_sparse_attention_cross_b200 as cba
    for n in (1, 2, 3, 5, 8, 10, 16, 33):
        for rho in (0.0, 0.1, 0.25, 0.3, 1 / 3, 0.5, 0.6, 0.7, 0.875, 0.9, 1.0):
            assert cba.min_votes_for(rho, n) == oracle.min_votes_for(rho, n), (rho, n)
    for nkb in (1, 7, 256, 350, 591):
        for frac in (1e-9, 0.1, 0.2, 0.25, 1 / 3, 0.5, 0.999, 1.0):
            assert cba.topk_count(frac, nkb) == oracle.topk_count(frac, nkb), (frac, nkb)
    out = ctypes.c_int32(0)
    assert lib.calibatt_topk_count(0.0, 10, ctypes.byref(out)) == _lib.E_INVALID
    assert lib.calibatt_min_votes(float("nan"), 4, ctypes.byref(out)) == _lib.E_INVALID
