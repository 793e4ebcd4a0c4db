"""Device-side failure detection without faulting the GPU.

A corrupt block list is caught by the kernels' own checks (status
CALIBATT_E_CORRUPT, affected rows written as 0 / -inf); a bounded wait on a
barrier that nothing completes gives up and reports CALIBATT_E_TIMEOUT; the
context stays usable afterwards.
"""

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import _lib
from block_sparse_attention_cross_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_corrupt_blocklist_reported(dtype):
    N = Np = 512
    H, d = 2, 128
    q, k, v = syn.normal_qkv(1, H, N, Np, d, 5)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    qd, kd, vd = (torch.from_numpy(x).cuda().to(tdt) for x in (q, k, v))
    mask = np.ones((H, 4, 4), np.uint8)
    bl = cba.compile(torch.from_numpy(mask).cuda())
    good = cba.sparse_attn_fwd(qd, kd, vd, bl, N)
    bl.row_base[3] = 7                    # row 3 now points past the last key block
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = cba.sparse_attn_fwd(qd, kd, vd, bl, N, return_lse=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == _lib.E_CORRUPT
    assert torch.all(o[0, 0, 3 * 128:4 * 128] == 0)
    assert torch.all(torch.isneginf(lse[0, 0, 3 * 128:4 * 128]))
    assert torch.equal(o[0, 1], good[0, 1])          # other rows untouched
    bl.row_base[3] = 0
    bl.pat_ptr[1] = 5                                   # pattern range now inverted
    status.zero_()
    cba.sparse_attn_fwd(qd, kd, vd, bl, N, status=status)
    torch.cuda.synchronize()
    assert status.item() == _lib.E_CORRUPT


def test_bounded_wait_times_out_cleanly():
    assert cba.selftest_wait_timeout(5_000_000) == _lib.E_TIMEOUT
    # the context is still healthy
    x = torch.ones(1024, device="cuda")
    assert float(x.sum().item()) == 1024.0


def test_unsupported_shapes_rejected():
    x = torch.zeros(1, 1, 256, 96, dtype=torch.bfloat16, device="cuda")
    bl = cba.compile(torch.ones((1, 2, 2), dtype=torch.uint8, device="cuda"))
    with pytest.raises(cba.CalibattError) as e:
        cba.sparse_attn_fwd(x, x, x, bl, 256)
    assert e.value.code == _lib.E_UNSUPPORTED
