"""Calibrated block-sparse spatiotemporal attention (CalibAtt) for B200.

Thin Python binding over libcalibatt.so (C ABI: ``include/calibatt.h``).
Every step of the computation runs in the library's CUDA kernels; this module
only checks and marshals arguments, allocates outputs and workspace with
PyTorch, and passes the current CUDA stream.  There is no CPU fallback: the
functions raise if the library is missing or a tensor is not on a GPU.

Method (arXiv 2603.05503, paper page): offline calibration scores key blocks
per query block by their post-softmax energy (Figure 2, Table S5), keeps the
top blocks (Figure 5(a)), votes them across calibration inputs with an
agreement threshold (Figure 3(b), Figure 7), compiles the result into
per-(layer, head, timestep) kept-block lists (Abstract), and at inference
computes only the kept blocks (Abstract, Figure 5(b) top).
"""

from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib
from ._lib import (BF16, DEDUP_HASH, DEDUP_HASH_WEAK, DEDUP_NONE, FP32, SELECT_ENERGY, SELECT_TOPK,
                   CalibattError, check, load)

__all__ = [
    "BlockList", "sparse_attn_fwd", "sparse_attn_fwd_qk", "sparse_attn_fwd_streamed", "block_energy", "timestep_clusters",
    "share_masks", "share_timesteps", "interval_counts", "merge_intervals", "skiplist_report", "gather_rows",
    "anchor_rows", "anchor_plan", "AnchorPlan", "anchor_attention", "spatial_similarity", "repetition_flags",
    "calibrate_schedule", "block_energy_noalloc", "select_vote", "finalize_mask", "calibrate",
    "compile", "compile_size", "selftest_wait_timeout", "min_votes_for", "topk_count", "launch_count",
    "default_scale", "CalibattError", "BF16", "FP32", "SELECT_TOPK", "SELECT_ENERGY",
    "DEDUP_NONE", "DEDUP_HASH", "DEDUP_HASH_WEAK", "load",
    "save_state", "load_state", "save_calibration", "load_calibration", "save_masks", "load_masks",
    "save_blocklist", "load_blocklist",
]


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}: use torch.bfloat16 or torch.float32")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _check_buf(name, t, shape, dtype):
    """Raises unless the caller-supplied buffer ``t`` (None: not given) has
    exactly ``shape`` and ``dtype``.  The library reads or writes that many
    elements through the bare pointer and cannot check the size itself."""
    if t is None:
        return
    if tuple(t.shape) != tuple(int(x) for x in shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} of shape {tuple(int(x) for x in shape)}, "
                         f"got {t.dtype} of shape {tuple(t.shape)}")


def _check_status(status):
    if status is not None and (status.dtype != torch.int32 or status.numel() < 1):
        raise ValueError("status must be an int32 tensor with at least one element")


def default_scale(d):
    """float32 of 1/sqrt(d): the softmax scale the kernels multiply by."""
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))


def launch_count():
    """Kernel launches issued by the library so far in this process."""
    return int(load().calibatt_launch_count())


def min_votes_for(rho, n_inputs):
    """Integer agreement threshold: keep a block iff votes / I >= rho (``calibatt_min_votes``)."""
    out = ctypes.c_int32(0)
    check(load().calibatt_min_votes(float(rho), int(n_inputs), ctypes.byref(out)))
    return out.value


def topk_count(frac, nkb):
    """Kept key blocks per row in top-k mode: ceil(frac * nkb) clamped to [1, nkb] (``calibatt_topk_count``)."""
    out = ctypes.c_int32(0)
    check(load().calibatt_topk_count(float(frac), int(nkb), ctypes.byref(out)))
    return out.value


@dataclass
class BlockList:
    """Compiled kept-block lists on the GPU (see ``calibatt_blocklist``)."""

    n_maps: int
    n_q_blocks: int
    n_k_blocks: int
    block_q: int
    block_k: int
    row_base: torch.Tensor
    row_pat: torch.Tensor
    pat_ptr: torch.Tensor
    pat_off: torch.Tensor
    csr_row_ptr: torch.Tensor | None
    csr_col: torch.Tensor | None
    n_pat: int
    nnz_pat: int
    nnz: int

    def as_struct(self):
        s = _lib.Blocklist()
        s.n_maps, s.n_q_blocks, s.n_k_blocks = self.n_maps, self.n_q_blocks, self.n_k_blocks
        s.block_q, s.block_k = self.block_q, self.block_k
        s.row_base = self.row_base.data_ptr()
        s.row_pat = self.row_pat.data_ptr()
        s.pat_ptr = self.pat_ptr.data_ptr()
        s.pat_off = self.pat_off.data_ptr() if self.pat_off.numel() else None
        s.csr_row_ptr = self.csr_row_ptr.data_ptr() if self.csr_row_ptr is not None else None
        s.csr_col = self.csr_col.data_ptr() if self.csr_col is not None and self.csr_col.numel() else None
        s.n_pat, s.nnz_pat, s.nnz = self.n_pat, self.nnz_pat, self.nnz
        return s

    def to_numpy(self):
        out = {k: getattr(self, k) for k in ("n_maps", "n_q_blocks", "n_k_blocks", "n_pat", "nnz_pat", "nnz")}
        for k in ("row_base", "row_pat", "pat_ptr", "pat_off", "csr_row_ptr", "csr_col"):
            v = getattr(self, k)
            out[k] = v.cpu().numpy() if v is not None else None
        return out

    @property
    def density(self):
        return self.nnz / float(self.n_maps * self.n_q_blocks * self.n_k_blocks)

    def kept_blocks(self, map_offset=0, n=None):
        """Kept blocks of maps [map_offset, map_offset + n) (``calibatt_blocklist_kept``; synchronizes)."""
        n = self.n_maps - map_offset if n is None else n
        dev = self.row_pat.device
        ws = torch.empty(1, dtype=torch.int64, device=dev)
        out = ctypes.c_int64(0)
        s = self.as_struct()
        with torch.cuda.device(dev):
            check(load().calibatt_blocklist_kept(ctypes.byref(s), int(map_offset), int(n), ctypes.byref(out), _ptr(ws),
                                                 8, _stream(dev)))
        return out.value


def sparse_attn_fwd(q, k, v, bl: BlockList, N, scale=None, map_offset=0, return_lse=False, out=None, lse=None,
                    status=None):
    """Block-sparse attention forward.  q, k, v: [B, H, Np, d] bf16 or fp32 on the GPU.

    Returns O (and LSE [B, H, Np] fp32 when ``return_lse``).  ``status`` is an
    optional int32 CUDA tensor that receives device-side error codes.
    """
    B, H, Np, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    _check_buf("out", out, q.shape, q.dtype)
    _check_buf("lse", lse, (B, H, Np), torch.float32)
    _check_status(status)
    _need_cuda(q, k, v)
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, H, Np), device=q.device, dtype=torch.float32)
    _need_cuda(out, lse, status)
    s = bl.as_struct()
    with torch.cuda.device(q.device):
        check(load().calibatt_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, int(N), Np, d,
                                              _dtype_code(q), scale, ctypes.byref(s), int(map_offset),
                                              _ptr(status), _stream(q.device)))
    return (out, lse) if return_lse else out


def sparse_attn_fwd_qk(q, k, v, bl: BlockList, Nq, Nk, scale=None, map_offset=0, return_lse=False, out=None,
                       lse=None, status=None):
    """Block-sparse attention forward with separate query and key lengths (bf16).

    q: [B, H, Npq, d] (Nq real rows); k, v: [B, H, Npk, d] (Nk real keys).
    ``bl`` has n_q_blocks = Npq / 128 and n_k_blocks = Npk / block_k, so the
    key padding follows the key-block size (any of 64, 80, 96, 128, 144)
    independently of the query blocks.  Returns O [B, H, Npq, d] (and LSE).
    """
    B, H, Npq, d = q.shape
    Npk = k.shape[2]
    if k.shape != (B, H, Npk, d) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("k, v must be [B, H, Npk, d] of q's dtype")
    _check_buf("out", out, q.shape, q.dtype)
    _check_buf("lse", lse, (B, H, Npq), torch.float32)
    _check_status(status)
    _need_cuda(q, k, v)
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, H, Npq), device=q.device, dtype=torch.float32)
    _need_cuda(out, lse, status)
    s = bl.as_struct()
    with torch.cuda.device(q.device):
        check(load().calibatt_sparse_attn_fwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, int(Nq), Npq,
                                                 int(Nk), Npk, d, _dtype_code(q), scale, ctypes.byref(s),
                                                 int(map_offset), _ptr(status), _stream(q.device)))
    return (out, lse) if return_lse else out


def _need_host(*ts):
    for t in ts:
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("host tensors must be contiguous CPU tensors (pin_memory() for overlap)")


def sparse_attn_fwd_streamed(q, k, v, bl: BlockList, N, staging, scale=None, map_offset=0, heads_per_chunk=2,
                             out=None, lse=None, status=None):
    """Block-sparse attention forward for q, k, v in host memory.

    q, k, v: [B, H, Np, d] bf16 or fp32 CPU tensors (pinned for overlap).
    ``staging``: (q_dev, k_dev, v_dev, o_dev[, lse_dev]) CUDA tensors of the
    same shapes, owned by the caller and overwritten.  Heads are processed in
    chunks of ``heads_per_chunk``; each chunk's host -> device copies, kernel
    and device -> host copy overlap those of the neighbouring chunks.  The
    result lands in ``out`` (a host tensor, allocated pinned when not given)
    and ``lse`` (host float32 [B, H, Np], only if given) once the current CUDA
    stream has been synchronised.  Returns ``out``.
    """
    _need_host(q, k, v, out, lse)
    B, H, Np, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    qd, kd, vd, od = staging[:4]
    lse_d = staging[4] if len(staging) > 4 else None
    if (lse is None) != (lse_d is None):
        raise ValueError("pass lse together with an lse staging buffer")
    for t in (qd, kd, vd, od):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("staging buffers must match q's shape and dtype")
    _check_buf("out", out, q.shape, q.dtype)
    _check_buf("lse", lse, (B, H, Np), torch.float32)
    _check_buf("lse staging buffer", lse_d, (B, H, Np), torch.float32)
    _check_status(status)
    _need_cuda(qd, kd, vd, od, lse_d, status)
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    s = bl.as_struct()
    with torch.cuda.device(qd.device):
        check(load().calibatt_sparse_attn_fwd_streamed(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(qd), _ptr(kd), _ptr(vd), _ptr(od), _ptr(lse_d),
            B, H, int(N), Np, d, _dtype_code(q), scale, ctypes.byref(s), int(map_offset), int(heads_per_chunk),
            _ptr(status), _stream(qd.device)))
    return out


def gather_rows(src, idx, rows_dst=None):
    """dst[..., i, :] = src[..., idx[i], :] over the leading dimensions (negative index: zero row)."""
    _need_cuda(src)
    idx_d = torch.as_tensor(idx, dtype=torch.int32).to(src.device).contiguous()
    rows_dst = idx_d.numel() if rows_dst is None else rows_dst
    lead = src.shape[:-2]
    planes = int(np.prod(lead)) if len(lead) else 1
    dst = torch.empty(tuple(lead) + (rows_dst, src.shape[-1]), dtype=src.dtype, device=src.device)
    row_bytes = src.shape[-1] * src.element_size()
    with torch.cuda.device(src.device):
        check(load().calibatt_gather_rows(_ptr(src), _ptr(dst), _ptr(idx_d), planes, src.shape[-2], rows_dst,
                                          row_bytes, _stream(src.device)))
    return dst


def anchor_rows(rows, k):
    """The k anchor rows of a frame of ``rows`` spatial rows, evenly spaced and
    centred, and for every row the anchor it takes its output from (the
    nearest, the lower one on a tie): ``calibatt_anchor_rows``."""
    anchors = np.zeros(int(k), dtype=np.int32)
    nearest = np.zeros(int(rows), dtype=np.int32)
    check(load().calibatt_anchor_rows(int(rows), int(k), anchors.ctypes.data_as(ctypes.c_void_p),
                                      nearest.ctypes.data_as(ctypes.c_void_p)))
    return anchors.tolist(), nearest.tolist()


@dataclass
class AnchorPlan:
    """Index lists of the spatial-repetition path for one video geometry."""
    N: int
    Np: int
    nq: int          # gathered anchor query tokens
    npq: int         # padded to a multiple of 128
    idx_q: torch.Tensor   # [npq] int32: source token of every gathered query (-1: padding)
    idx_o: torch.Tensor   # [Np] int32: gathered row every token's output comes from (-1: padding)


def anchor_plan(frames, rows, cols, k_anchor, Np, device):
    """Plan of :func:`anchor_attention` for a frames x rows x cols video padded
    to Np tokens: ``calibatt_anchor_plan`` on the device."""
    lib = load()
    nq, npq = ctypes.c_int(0), ctypes.c_int(0)
    check(lib.calibatt_anchor_plan_size(int(frames), int(rows), int(cols), int(k_anchor), ctypes.byref(nq),
                                        ctypes.byref(npq)))
    device = torch.device(device)
    if device.type != "cuda":
        raise ValueError("the anchor plan is computed on a CUDA device")
    idx_q = torch.empty(npq.value, dtype=torch.int32, device=device)
    idx_o = torch.empty(int(Np), dtype=torch.int32, device=device)
    with torch.cuda.device(device):
        check(lib.calibatt_anchor_plan(int(frames), int(rows), int(cols), int(k_anchor), int(Np), _ptr(idx_q),
                                       _ptr(idx_o), _stream(device)))
    return AnchorPlan(int(frames) * int(rows) * int(cols), int(Np), nq.value, npq.value, idx_q, idx_o)


def anchor_attention(q, k, v, plan: AnchorPlan, bl=None, scale=None):
    """Spatial-repetition attention (paper page, Figure 4, Figure 5(b) bottom,
    Table S4): attention is computed only for the query tokens of the plan's
    anchor rows (k evenly spaced spatial rows per frame) against all keys, and
    every token takes the output of the token in the same frame and column on
    its nearest anchor row.

    q, k, v: [B, H, Np, d] bf16 CUDA tensors.  ``bl``: block list over the
    gathered queries (n_q_blocks = plan.npq / 128, n_k_blocks = Np / block_k);
    dense (every key block) when None.  Returns O [B, H, Np, d].
    """
    _need_cuda(q, k, v)
    B, H, Np, d = q.shape
    qg = gather_rows(q, plan.idx_q)
    if bl is None:
        bl = compile(torch.ones((H, plan.npq // 128, Np // 128), dtype=torch.uint8, device=q.device))
    scale = default_scale(d) if scale is None else float(scale)
    og = torch.empty_like(qg)
    s = bl.as_struct()
    with torch.cuda.device(q.device):
        check(load().calibatt_sparse_attn_fwd_qk(_ptr(qg), _ptr(k), _ptr(v), _ptr(og), None, B, H, plan.nq, plan.npq,
                                                 int(plan.N), Np, d, _dtype_code(q), scale, ctypes.byref(s), 0, None,
                                                 _stream(q.device)))
    return gather_rows(og, plan.idx_o)


def spatial_similarity(q, k, N, frames, rows, cols, scale=None, status=None):
    """Spatial-similarity score [H] float32 of one input (``calibatt_spatial_similarity``).

    q, k: [H, Np, d] bf16 CUDA tensors; the first frames x rows x cols tokens
    are the video.  The score of a head is the mean cosine similarity of the
    dense attention rows of vertically adjacent query tokens (same frame and
    column): near 1 for maps that repeat across spatial rows (paper page,
    Figure 4, Figure 6(a), Figure S13).
    """
    H, Np, d = q.shape
    if k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must share shape and dtype")
    _check_status(status)
    _need_cuda(q, k)
    scale = default_scale(d) if scale is None else float(scale)
    n = ctypes.c_size_t(0)
    check(load().calibatt_spatial_similarity_workspace_size(H, Np, ctypes.byref(n)))
    ws = torch.empty(n.value, dtype=torch.uint8, device=q.device)
    out = torch.empty(H, dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        check(load().calibatt_spatial_similarity(_ptr(q), _ptr(k), H, int(N), Np, d, _dtype_code(q), int(frames),
                                                 int(rows), int(cols), scale, _ptr(out), _ptr(ws), ws.nbytes,
                                                 _ptr(status), _stream(q.device)))
    return out


def repetition_flags(scores, tau=0.87):
    """Repetition dictionary (``calibatt_repetition_flags``): from per-input
    scores [n_inputs, n_maps] float32 (CUDA), the mean score per map and the
    flags mean >= tau (paper page, Figure 5(a), Figure S13: tau = 0.87)."""
    if scores.dim() != 2 or scores.dtype != torch.float32:
        raise ValueError("scores must be float32 [n_inputs, n_maps]")
    _need_cuda(scores)
    n_inputs, n_maps = scores.shape
    mean = torch.empty(n_maps, dtype=torch.float32, device=scores.device)
    flags = torch.empty(n_maps, dtype=torch.uint8, device=scores.device)
    with torch.cuda.device(scores.device):
        check(load().calibatt_repetition_flags(_ptr(scores), n_inputs, n_maps, float(tau), _ptr(mean), _ptr(flags),
                                               _stream(scores.device)))
    return mean, flags


def _calib_workspace(H, N, Np, d, bq, bk, device):
    n = ctypes.c_size_t(0)
    check(load().calibatt_calibrate_workspace_size(H, int(N), Np, d, bq, bk, ctypes.byref(n)))
    return torch.empty(n.value, dtype=torch.uint8, device=device)


def block_energy(q, k, N, block_q=128, block_k=128, scale=None, status=None, workspace=None):
    """Block energies [H, nqb, nkb] fp32 of one input; q, k: [H, Np, d]."""
    H, Np, d = q.shape
    if k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must share shape and dtype")
    _check_status(status)
    _need_cuda(q, k, workspace)
    scale = default_scale(d) if scale is None else float(scale)
    E = torch.empty((H, Np // block_q, -(-int(N) // block_k)), device=q.device, dtype=torch.float32)
    ws = _calib_workspace(H, N, Np, d, block_q, block_k, q.device) if workspace is None else workspace
    with torch.cuda.device(q.device):
        check(load().calibatt_block_energy(_ptr(q), _ptr(k), H, int(N), Np, d, _dtype_code(q), block_q, block_k,
                                           scale, _ptr(E), _ptr(ws), ws.nbytes, _ptr(status), _stream(q.device)))
    return E


def block_energy_noalloc(q, k, N, block_q=128, block_k=128, scale=None, status=None, out=None):
    """Block energies like :func:`block_energy`, without any device allocation by the library.

    For callers that cannot hand the library a workspace: the per-row scratch
    lives in a fixed 16 MiB array inside the library (H * Np <= 4 Mi rows).
    Calls that overlap on the GPU share that array and must not be issued.
    Pass ``out`` ([H, nqb, nkb] float32) to avoid the one allocation this
    wrapper would otherwise make for the result.
    """
    H, Np, d = q.shape
    if k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must share shape and dtype")
    eshape = (H, Np // block_q, -(-int(N) // block_k))
    _check_buf("out", out, eshape, torch.float32)
    _check_status(status)
    _need_cuda(q, k)
    scale = default_scale(d) if scale is None else float(scale)
    E = torch.empty(eshape, device=q.device, dtype=torch.float32) if out is None else out
    _need_cuda(E, status)
    with torch.cuda.device(q.device):
        check(load().calibatt_block_energy_noalloc(_ptr(q), _ptr(k), H, int(N), Np, d, _dtype_code(q), block_q,
                                                   block_k, scale, _ptr(E), _ptr(status), _stream(q.device)))
    return E


def select_vote(energy, mode, param, votes, energy_sum):
    """Adds one input's selection (top-k fraction or energy eps) into votes / energy_sum (in place)."""
    if energy.dim() != 3 or energy.dtype != torch.float32:
        raise ValueError("energy must be float32 [H, nqb, nkb]")
    H, nqb, nkb = energy.shape
    _check_buf("votes", votes, energy.shape, torch.int32)
    _check_buf("energy_sum", energy_sum, energy.shape, torch.float32)
    _need_cuda(energy, votes, energy_sum)
    with torch.cuda.device(energy.device):
        check(load().calibatt_select_vote(_ptr(energy), H, nqb, nkb, int(mode), float(param), _ptr(votes),
                                          _ptr(energy_sum), _stream(energy.device)))
    return votes, energy_sum


def finalize_mask(votes, energy_sum, min_votes):
    """uint8 mask [H, nqb, nkb] = votes >= min_votes, with the empty-row guard."""
    if votes.dim() != 3 or votes.dtype != torch.int32:
        raise ValueError("votes must be int32 [H, nqb, nkb]")
    _check_buf("energy_sum", energy_sum, votes.shape, torch.float32)
    _need_cuda(votes, energy_sum)
    H, nqb, nkb = votes.shape
    mask = torch.empty((H, nqb, nkb), dtype=torch.uint8, device=votes.device)
    with torch.cuda.device(votes.device):
        check(load().calibatt_finalize_mask(_ptr(votes), _ptr(energy_sum), H, nqb, nkb, int(min_votes), _ptr(mask),
                                            _stream(votes.device)))
    return mask


def calibrate(q_list, k_list, N, block_q=128, block_k=128, scale=None, select_mode=SELECT_TOPK, select_param=0.25,
              rho=0.5, min_votes=None, votes=None, energy_sum=None, finalize=True, status=None, inputs_before=0):
    """Calibration pass.  Returns (mask or None, votes, energy_sum).

    ``votes`` / ``energy_sum`` (int32 / fp32 [H, nqb, nkb]) accumulate across
    calls, so calibration can resume: pass the state after ``inputs_before``
    earlier inputs (see :mod:`.dictionary` for saving it).  ``min_votes``
    defaults to ceil(rho * I) with I = inputs_before + len(q_list), the total
    number of inputs behind the votes.
    """
    n = len(q_list)
    if n != len(k_list) or n == 0:
        raise ValueError("need the same non-zero number of q and k tensors")
    if int(inputs_before) < 0 or (int(inputs_before) > 0 and (votes is None or energy_sum is None)):
        raise ValueError("inputs_before > 0 needs the votes and energy_sum of those inputs")
    H, Np, d = q_list[0].shape
    for t in (*q_list, *k_list):
        if t.shape != q_list[0].shape or t.dtype != q_list[0].dtype or t.device != q_list[0].device:
            raise ValueError("every q and k must share shape, dtype and device")
    dev = q_list[0].device
    nqb, nkb = Np // block_q, -(-int(N) // block_k)
    _check_buf("votes", votes, (H, nqb, nkb), torch.int32)
    _check_buf("energy_sum", energy_sum, (H, nqb, nkb), torch.float32)
    _check_status(status)
    _need_cuda(*q_list, *k_list, votes, energy_sum)
    scale = default_scale(d) if scale is None else float(scale)
    if votes is None:
        votes = torch.zeros((H, nqb, nkb), dtype=torch.int32, device=dev)
    if energy_sum is None:
        energy_sum = torch.zeros((H, nqb, nkb), dtype=torch.float32, device=dev)
    if min_votes is None:
        min_votes = min_votes_for(rho, int(inputs_before) + n)
    mask = torch.empty((H, nqb, nkb), dtype=torch.uint8, device=dev) if finalize else None
    ws = _calib_workspace(H, N, Np, d, block_q, block_k, dev)
    qp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in q_list])
    kp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in k_list])
    with torch.cuda.device(dev):
        check(load().calibatt_calibrate(qp, kp, n, H, int(N), Np, d, _dtype_code(q_list[0]), block_q, block_k, scale,
                                        int(select_mode), float(select_param), _ptr(votes), _ptr(energy_sum),
                                        int(min_votes), _ptr(mask), _ptr(ws), ws.nbytes, _ptr(status),
                                        _stream(dev)))
    return mask, votes, energy_sum


def timestep_clusters(masks, tau):
    """Runs of alike consecutive timesteps per layer (synchronizes).

    ``masks``: uint8 [L, T, H, nqb, nkb] CUDA tensor.  Returns (run_of, n_runs):
    run_of an int32 [L, T] CPU tensor of global run indices in (layer, time)
    order, n_runs their number.
    """
    _need_cuda(masks)
    if masks.dtype != torch.uint8 or masks.dim() != 5:
        raise ValueError("masks must be uint8 [L, T, H, nqb, nkb]")
    L, T, H, nqb, nkb = masks.shape
    n = ctypes.c_size_t(0)
    check(load().calibatt_timestep_clusters_workspace_size(L, T, H, ctypes.byref(n)))
    ws = torch.empty(max(int(n.value), 1), dtype=torch.uint8, device=masks.device)
    run_of = torch.empty((L, T), dtype=torch.int32)
    n_runs = ctypes.c_int32(0)
    with torch.cuda.device(masks.device):
        check(load().calibatt_timestep_clusters(_ptr(masks), L, T, H, nqb, nkb, float(tau), _ptr(run_of),
                                                ctypes.byref(n_runs), _ptr(ws), ws.numel(), _stream(masks.device)))
    return run_of, n_runs.value


def share_masks(masks, run_of, n_runs):
    """Union masks [n_runs, H, nqb, nkb] uint8 of the runs ``run_of`` ([L, T] int32)."""
    if masks.dtype != torch.uint8 or masks.dim() != 5:
        raise ValueError("masks must be uint8 [L, T, H, nqb, nkb]")
    L, T, H, nqb, nkb = masks.shape
    if tuple(run_of.shape) != (L, T):
        raise ValueError(f"run_of must have shape {(L, T)}, got {tuple(run_of.shape)}")
    _need_cuda(masks)
    run_dev = run_of.to(device=masks.device, dtype=torch.int32).contiguous()
    shared = torch.empty((int(n_runs), H, nqb, nkb), dtype=torch.uint8, device=masks.device)
    with torch.cuda.device(masks.device):
        check(load().calibatt_share_masks(_ptr(masks), L, T, H, nqb, nkb, _ptr(run_dev), int(n_runs), _ptr(shared),
                                          _stream(masks.device)))
    return shared


def share_timesteps(masks, tau):
    """Timestep sharing of a [L, T, H, nqb, nkb] mask dictionary.

    Returns (shared masks [n_runs * H, nqb, nkb] ready for :func:`compile`,
    map_offset [L, T] int64 CPU tensor: the ``map_offset`` of call (l, t)).
    """
    run_of, n_runs = timestep_clusters(masks, tau)
    shared = share_masks(masks, run_of, n_runs)
    H = masks.shape[2]
    return shared.reshape(n_runs * H, *masks.shape[3:]), run_of.to(torch.int64) * H


def interval_counts(masks):
    """int32 [n_maps, nqb]: kept-block intervals of every row of uint8 masks [n_maps, nqb, nkb]."""
    if masks.dtype != torch.uint8 or masks.dim() != 3:
        raise ValueError("masks must be uint8 [n_maps, nqb, nkb]")
    _need_cuda(masks)
    n_maps, nqb, nkb = masks.shape
    counts = torch.empty((n_maps, nqb), dtype=torch.int32, device=masks.device)
    with torch.cuda.device(masks.device):
        check(load().calibatt_interval_counts(_ptr(masks), n_maps, nqb, nkb, _ptr(counts), _stream(masks.device)))
    return counts


def merge_intervals(masks, width_per_map):
    """Merges, in place, every row of map i to at most width_per_map[i] intervals.

    Returns the number of filled blocks (synchronizes)."""
    if masks.dtype != torch.uint8 or masks.dim() != 3:
        raise ValueError("masks must be uint8 [n_maps, nqb, nkb]")
    n_maps, nqb, nkb = masks.shape
    if torch.as_tensor(width_per_map).numel() != n_maps:
        raise ValueError(f"width_per_map must have one entry per map ({n_maps})")
    _need_cuda(masks)
    width = torch.as_tensor(width_per_map, dtype=torch.int32).to(masks.device).contiguous()
    filled = torch.zeros(1, dtype=torch.int64, device=masks.device)
    with torch.cuda.device(masks.device):
        check(load().calibatt_merge_intervals(_ptr(masks), n_maps, nqb, nkb, _ptr(width), _ptr(filled),
                                              _stream(masks.device)))
    return int(filled.item())


def skiplist_report(masks, maps_per_layer, pcts=(100.0, 99.0, 95.0)):
    """Storage of a mask dictionary [n_maps, nqb, nkb] in the paper page's
    padded per-layer interval skip lists (one interval = an int32 pair) next
    to this library's compiled forms.

    Per layer: full allocation (ceil(nkb / 2) intervals per row), trimmed to
    the widest row, and merged at each percentile in ``pcts`` (nearest rank of
    the layer's interval counts; outlier rows merged by
    :func:`merge_intervals`, whose filled blocks lower the sparsity).  Sizes
    from ``calibatt_skiplist_sizes`` and ``calibatt_blocklist_bytes``;
    synchronizes.
    """
    lib = load()
    n_maps, nqb, nkb = masks.shape
    if n_maps % maps_per_layer:
        raise ValueError("n_maps must be a multiple of maps_per_layer")
    dev = masks.device
    counts = interval_counts(masks)
    layers = n_maps // maps_per_layer

    def sizes(mpl, pc):
        nl = n_maps // mpl
        n = ctypes.c_size_t(0)
        check(lib.calibatt_skiplist_sizes_workspace_size(n_maps, mpl, len(pc), ctypes.byref(n)))
        ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
        pc_h = np.asarray(pc, dtype=np.float64)
        layer_max = np.zeros(nl, dtype=np.int32)
        layer_width = np.zeros(max(1, len(pc) * nl), dtype=np.int32)
        map_width = torch.empty(max(1, len(pc) * n_maps), dtype=torch.int32, device=dev)
        nbytes = np.zeros(2 + len(pc), dtype=np.int64)
        with torch.cuda.device(dev):
            check(lib.calibatt_skiplist_sizes(_ptr(counts), n_maps, nqb, nkb, mpl,
                                              pc_h.ctypes.data_as(ctypes.c_void_p), len(pc),
                                              layer_max.ctypes.data_as(ctypes.c_void_p),
                                              layer_width.ctypes.data_as(ctypes.c_void_p), _ptr(map_width),
                                              nbytes.ctypes.data_as(ctypes.c_void_p), _ptr(ws), ws.numel(),
                                              _stream(dev)))
        return layer_max, layer_width, map_width, nbytes

    layer_max, layer_width, map_width, nbytes = sizes(maps_per_layer, pcts)
    g_max, g_p95, _, _ = sizes(n_maps, (95.0,))   # the whole dictionary as one group: max and p95
    nnz, n_pat, nnz_pat = compile_size(masks)
    cells = float(n_maps * nqb * nkb)
    out = {"rows": n_maps * nqb, "kept_blocks": nnz, "density": nnz / cells,
           "intervals_max": int(g_max[0]), "intervals_p95": int(g_p95[0]),
           "skiplist_full_bytes": int(nbytes[0]), "skiplist_trimmed_bytes": int(nbytes[1]),
           "layer_max": layer_max.tolist(), "merged": []}
    for p, pct in enumerate(pcts):
        m = masks.clone()
        filled = merge_intervals(m, map_width[p * n_maps:(p + 1) * n_maps])
        out["merged"].append({"pct": pct, "bytes": int(nbytes[2 + p]), "filled_blocks": filled,
                              "layer_width": layer_width[p * layers:(p + 1) * layers].tolist(),
                              "density": (nnz + filled) / cells})
        del m
    csr, pool = ctypes.c_int64(0), ctypes.c_int64(0)
    check(lib.calibatt_blocklist_bytes(n_maps, nqb, int(nnz), int(n_pat), int(nnz_pat), ctypes.byref(csr),
                                       ctypes.byref(pool)))
    out["csr_bytes"] = csr.value
    out["pattern_pool_bytes"] = pool.value
    return out


def calibrate_schedule(inputs_per_step, N, param_of, select_mode=SELECT_ENERGY, rho=0.5, **kw):
    """Calibration of every denoising step with its own selection parameter.

    The paper page's energy threshold is a function of the normalized
    timestep (Figure S8: epsilon against t/T; the values are not printed, so
    the caller supplies them).  ``inputs_per_step``: for steps t = 0 .. T-1,
    a pair (q_list, k_list) of that step's calibration inputs ([H, Np, d]
    CUDA tensors); ``param_of(t, T)``: the selection parameter of step t
    (epsilon for SELECT_ENERGY, the kept fraction for SELECT_TOPK).  Returns
    uint8 masks [T, H, nqb, nkb], one :func:`calibrate` per step.
    """
    T = len(inputs_per_step)
    masks = []
    for t, (q_list, k_list) in enumerate(inputs_per_step):
        m, _, _ = calibrate(q_list, k_list, N, select_mode=select_mode, select_param=float(param_of(t, T)), rho=rho,
                            **kw)
        masks.append(m)
    return torch.stack(masks)


def _compile_ws(n_maps, nqb, nkb, dev):
    n = ctypes.c_size_t(0)
    check(load().calibatt_compile_workspace_size(n_maps, nqb, nkb, ctypes.byref(n)))
    return torch.empty(n.value, dtype=torch.uint8, device=dev)


def compile_size(masks, dedup=DEDUP_HASH, workspace=None):
    """(nnz, n_pat, nnz_pat) of compiling ``masks`` [n_maps, nqb, nkb] uint8 (synchronizes)."""
    if masks.dtype != torch.uint8 or masks.dim() != 3:
        raise ValueError("masks must be uint8 [n_maps, nqb, nkb]")
    _need_cuda(masks, workspace)
    n_maps, nqb, nkb = masks.shape
    ws = _compile_ws(n_maps, nqb, nkb, masks.device) if workspace is None else workspace
    nnz, n_pat, nnz_pat = ctypes.c_int64(0), ctypes.c_int32(0), ctypes.c_int32(0)
    with torch.cuda.device(masks.device):
        check(load().calibatt_compile_size(_ptr(masks), n_maps, nqb, nkb, int(dedup), ctypes.byref(nnz),
                                           ctypes.byref(n_pat), ctypes.byref(nnz_pat), _ptr(ws), ws.nbytes,
                                           _stream(masks.device)))
    return nnz.value, n_pat.value, nnz_pat.value


def compile(masks, block_q=128, block_k=128, dedup=DEDUP_HASH, with_csr=True):
    """Compiles uint8 masks [n_maps, nqb, nkb] into a :class:`BlockList` (synchronizes)."""
    if masks.dtype != torch.uint8 or masks.dim() != 3:
        raise TypeError("masks must be uint8 [n_maps, nqb, nkb]")
    _need_cuda(masks)
    n_maps, nqb, nkb = masks.shape
    dev = masks.device
    ws = _compile_ws(n_maps, nqb, nkb, dev)
    nnz, n_pat, nnz_pat = compile_size(masks, dedup, ws)
    R = n_maps * nqb
    bl = BlockList(
        n_maps, nqb, nkb, block_q, block_k,
        row_base=torch.empty(R, dtype=torch.int32, device=dev),
        row_pat=torch.empty(R, dtype=torch.int32, device=dev),
        pat_ptr=torch.empty(n_pat + 1, dtype=torch.int32, device=dev),
        pat_off=torch.empty(max(nnz_pat, 1), dtype=torch.int16, device=dev)[:nnz_pat],
        csr_row_ptr=torch.empty(R + 1, dtype=torch.int64, device=dev) if with_csr else None,
        csr_col=torch.empty(max(nnz, 1), dtype=torch.int16, device=dev)[:nnz] if with_csr else None,
        n_pat=n_pat, nnz_pat=nnz_pat, nnz=nnz,
    )
    s = bl.as_struct()
    if nnz_pat == 0:
        s.pat_off = None
    with torch.cuda.device(dev):
        check(load().calibatt_compile(_ptr(masks), n_maps, nqb, nkb, int(dedup), block_q, block_k, ctypes.byref(s),
                                      _ptr(ws), ws.nbytes, _stream(dev)))
    return bl


def selftest_wait_timeout(limit_ns=10_000_000, device=None):
    """Runs the never-completing bounded wait; returns the device status (CALIBATT_E_TIMEOUT expected)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(load().calibatt_selftest_wait_timeout(int(limit_ns), _ptr(status), _stream(dev)))
    return int(status.item())


from .dictionary import (load_blocklist, load_calibration, load_masks, load_state, save_blocklist,  # noqa: E402
                         save_calibration, save_masks, save_state)
