"""Caller-supplied buffers of the Python binding are checked before any call
into the library: the C ABI takes bare pointers and reads or writes as many
elements as the sizes say, so a buffer of the wrong shape or dtype must be
rejected on the host.  CPU only: every case fails before a device is needed,
and a well-formed call on CPU tensors reaches the "must be CUDA" check."""

import pytest
import torch

import block_sparse_attention_cross_b200 as cba


def _qkv(B=1, H=2, Np=256, d=64, dtype=torch.bfloat16):
    return [torch.zeros(B, H, Np, d, dtype=dtype) for _ in range(3)]


def test_fwd_out_and_lse_shapes():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="out must be"):
        cba.sparse_attn_fwd(q, k, v, None, 250, out=torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out must be"):
        cba.sparse_attn_fwd(q, k, v, None, 250, out=torch.zeros_like(q, dtype=torch.float32))
    with pytest.raises(ValueError, match="lse must be"):
        cba.sparse_attn_fwd(q, k, v, None, 250, lse=torch.zeros(1, 2, 255))
    with pytest.raises(ValueError, match="status must be"):
        cba.sparse_attn_fwd(q, k, v, None, 250, status=torch.zeros(0, dtype=torch.int32))
    with pytest.raises(ValueError, match="status must be"):
        cba.sparse_attn_fwd(q, k, v, None, 250, status=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA"):
        cba.sparse_attn_fwd(q, k, v, None, 250, out=torch.zeros_like(q), lse=torch.zeros(1, 2, 256))


def test_fwd_qk_out_shape():
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="out must be"):
        cba.sparse_attn_fwd_qk(q, k, k, None, 100, 250, out=torch.zeros_like(k))
    with pytest.raises(ValueError, match="lse must be"):
        cba.sparse_attn_fwd_qk(q, k, k, None, 100, 250, lse=torch.zeros(1, 2, 256))


def test_streamed_buffers():
    q, k, v = _qkv()
    staging = [torch.zeros_like(q) for _ in range(4)]
    with pytest.raises(ValueError, match="out must be"):
        cba.sparse_attn_fwd_streamed(q, k, v, None, 250, staging, out=torch.zeros(1, 2, 256, 32, dtype=q.dtype))
    with pytest.raises(ValueError, match="lse must be"):
        cba.sparse_attn_fwd_streamed(q, k, v, None, 250, staging + [torch.zeros(1, 2, 256)],
                                     lse=torch.zeros(1, 2, 128))
    with pytest.raises(ValueError, match="lse staging buffer must be"):
        cba.sparse_attn_fwd_streamed(q, k, v, None, 250, staging + [torch.zeros(2, 256)], lse=torch.zeros(1, 2, 256))


def test_energy_buffers():
    q = torch.zeros(2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="share shape"):
        cba.block_energy(q, torch.zeros(2, 128, 64, dtype=torch.bfloat16), 250)
    with pytest.raises(ValueError, match="out must be"):
        # 250 real keys in blocks of 80 -> 4 key blocks, not 2
        cba.block_energy_noalloc(q, q, 250, block_k=80, out=torch.zeros(2, 2, 2))
    with pytest.raises(ValueError, match="CUDA"):
        cba.block_energy_noalloc(q, q, 250, block_k=80, out=torch.zeros(2, 2, 4))


def test_select_vote_and_finalize_buffers():
    e = torch.zeros(2, 3, 5)
    with pytest.raises(ValueError, match="votes must be"):
        cba.select_vote(e, cba.SELECT_TOPK, 0.25, torch.zeros(2, 3, 4, dtype=torch.int32), torch.zeros(2, 3, 5))
    with pytest.raises(ValueError, match="energy_sum must be"):
        cba.select_vote(e, cba.SELECT_TOPK, 0.25, torch.zeros(2, 3, 5, dtype=torch.int32), torch.zeros(2, 3, 5,
                                                                                                    dtype=torch.float64))
    with pytest.raises(ValueError, match="energy must be"):
        cba.select_vote(e.double(), cba.SELECT_TOPK, 0.25, None, None)
    with pytest.raises(ValueError, match="energy_sum must be"):
        cba.finalize_mask(torch.zeros(2, 3, 5, dtype=torch.int32), torch.zeros(2, 3, 6), 1)
    with pytest.raises(ValueError, match="votes must be"):
        cba.finalize_mask(torch.zeros(2, 3, 5), torch.zeros(2, 3, 5), 1)


def test_calibrate_inputs_must_agree():
    q = torch.zeros(2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="share shape"):
        cba.calibrate([q, torch.zeros(2, 128, 64, dtype=torch.bfloat16)], [q, q], 250)
    with pytest.raises(ValueError, match="share shape"):
        cba.calibrate([q, q], [q, q.float()], 250)
    with pytest.raises(ValueError, match="votes must be"):
        cba.calibrate([q], [q], 250, votes=torch.zeros(2, 2, 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        cba.calibrate([q], [q], 250, votes=torch.zeros(2, 2, 2, dtype=torch.int32))


def test_mask_tools_shapes():
    m = torch.zeros(4, 3, 5, dtype=torch.uint8)
    with pytest.raises(ValueError, match="one entry per map"):
        cba.merge_intervals(m, [1, 2, 3])
    with pytest.raises(ValueError, match="uint8"):
        cba.interval_counts(m.int())
    with pytest.raises(ValueError, match="uint8"):
        cba.compile_size(m.bool())
    with pytest.raises(TypeError, match="uint8"):
        cba.compile(m[0])
    with pytest.raises(ValueError, match="run_of must have shape"):
        cba.share_masks(torch.zeros(2, 3, 1, 3, 5, dtype=torch.uint8), torch.zeros(3, 2, dtype=torch.int32), 2)
    with pytest.raises(ValueError, match="scores must be"):
        cba.repetition_flags(torch.zeros(4))
    with pytest.raises(ValueError, match="share shape"):
        cba.spatial_similarity(torch.zeros(2, 256, 64), torch.zeros(2, 256, 128), 250, 1, 5, 50)
