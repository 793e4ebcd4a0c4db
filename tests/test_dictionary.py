"""Saved calibration state, mask dictionaries and compiled block lists:
exact round trips, refusal of altered files, and the resume arguments of
``calibrate`` (CPU; the GPU resume test is in test_gpu_calibrate.py)."""

import io
import json
import zipfile

import numpy as np
import pytest
import torch

import block_sparse_attention_cross_b200 as cba
from block_sparse_attention_cross_b200 import dictionary


def test_round_trip_is_exact(tmp_path):
    rng = np.random.default_rng(3)
    arrays = {
        "m": torch.from_numpy((rng.random((4, 3, 5)) < 0.4).astype(np.uint8)),
        "v": torch.from_numpy(rng.integers(0, 9, (4, 3, 5)).astype(np.int32)),
        "e": torch.from_numpy(rng.random((4, 3, 5)).astype(np.float32)),
        "off": torch.from_numpy(rng.integers(-500, 500, 17).astype(np.int16)),
        "ptr": torch.arange(13, dtype=torch.int64),
        "empty": torch.empty(0, dtype=torch.int16),
        "f64": rng.random(6),
    }
    meta = {"block_q": 128, "block_k": 80, "rho": 0.5, "select": ["topk", 0.25]}
    p = tmp_path / "state.npz"
    dictionary.save_state(p, arrays, meta)
    got, gmeta = dictionary.load_state(p)
    assert gmeta == meta
    assert set(got) == set(arrays)
    for k, t in arrays.items():
        want = torch.as_tensor(t)
        assert got[k].dtype == want.dtype and got[k].shape == want.shape
        assert torch.equal(got[k], want)


def _rewrite(path, fn):
    """Rewrites the archive with fn(name, bytes) -> bytes applied to each member."""
    with zipfile.ZipFile(path) as z:
        members = {n: z.read(n) for n in z.namelist()}
    with zipfile.ZipFile(path, "w") as z:
        for n, b in members.items():
            z.writestr(n, fn(n, b))


def _npy_bytes(a):
    buf = io.BytesIO()
    np.save(buf, a)
    return buf.getvalue()


def test_altered_arrays_are_refused(tmp_path):
    p = tmp_path / "s.npz"
    votes = torch.arange(24, dtype=torch.int32).reshape(2, 3, 4)
    dictionary.save_state(p, {"votes": votes})
    # one vote changed, shape and dtype kept: the digest catches it
    changed = votes.numpy().copy()
    changed[1, 2, 3] += 1
    _rewrite(p, lambda n, b: _npy_bytes(changed) if n == "votes.npy" else b)
    with pytest.raises(ValueError, match="SHA-256"):
        dictionary.load_state(p)
    # a different shape
    dictionary.save_state(p, {"votes": votes})
    _rewrite(p, lambda n, b: _npy_bytes(votes.numpy().reshape(6, 4)) if n == "votes.npy" else b)
    with pytest.raises(ValueError, match="header says"):
        dictionary.load_state(p)
    # an array the header does not list
    dictionary.save_state(p, {"votes": votes})
    with zipfile.ZipFile(p, "a") as z:
        z.writestr("extra.npy", _npy_bytes(np.zeros(2, dtype=np.int32)))
    with pytest.raises(ValueError, match="do not match the header"):
        dictionary.load_state(p)


def test_format_and_names(tmp_path):
    p = tmp_path / "s.npz"
    dictionary.save_state(p, {"a": np.zeros(3, dtype=np.int32)})

    def other_format(n, b):
        if n != "__header__.npy":
            return b
        h = json.loads(bytes(np.load(io.BytesIO(b))).decode())
        h["format"] = "calibatt-state/0"
        return _npy_bytes(np.frombuffer(json.dumps(h).encode(), dtype=np.uint8))

    _rewrite(p, other_format)
    with pytest.raises(ValueError, match="format"):
        dictionary.load_state(p)
    with pytest.raises(ValueError, match="identifier"):
        dictionary.save_state(p, {"__header__": np.zeros(1, dtype=np.uint8)})
    with pytest.raises(TypeError, match="bfloat16"):
        dictionary.save_state(p, {"q": torch.zeros(2, dtype=torch.bfloat16)})
    with pytest.raises(TypeError, match="dtype"):
        dictionary.save_state(p, {"b": np.zeros(2, dtype=bool)})


def test_calibration_and_masks_helpers(tmp_path):
    votes = torch.randint(0, 5, (2, 3, 4), dtype=torch.int32)
    esum = torch.rand(2, 3, 4)
    p = tmp_path / "calib.npz"
    cba.save_calibration(p, votes, esum, 4, block_q=128, block_k=128, rho=0.5)
    v, e, n, meta = cba.load_calibration(p)
    assert torch.equal(v, votes) and torch.equal(e, esum) and n == 4
    assert meta["block_k"] == 128 and meta["rho"] == 0.5
    with pytest.raises(ValueError, match="not a mask dictionary"):
        cba.load_masks(p)
    with pytest.raises(ValueError, match="int32"):
        cba.save_calibration(p, votes.float(), esum, 4)
    with pytest.raises(ValueError, match="inputs_seen"):
        cba.save_calibration(p, votes, esum, 0)
    masks = (torch.rand(6, 3, 4) < 0.5).to(torch.uint8)
    q = tmp_path / "masks.npz"
    cba.save_masks(q, masks, layers=2, timesteps=1, heads=3)
    m, meta = cba.load_masks(q)
    assert torch.equal(m, masks) and meta["heads"] == 3
    with pytest.raises(ValueError, match="not a calibration state"):
        cba.load_calibration(q)


def _cpu_blocklist(with_csr):
    # a hand-built list of 2 maps x 2 query blocks over 5 key blocks: rows
    # {0, 1}, {}, {2, 3}, {1, 2} -> patterns [0, 1] (rows 0, 2, 3 share it)
    return cba.BlockList(
        2, 2, 5, 128, 128,
        row_base=torch.tensor([0, 0, 2, 1], dtype=torch.int32),
        row_pat=torch.tensor([1, 0, 1, 1], dtype=torch.int32),
        pat_ptr=torch.tensor([0, 0, 2], dtype=torch.int32),
        pat_off=torch.tensor([0, 1], dtype=torch.int16),
        csr_row_ptr=torch.tensor([0, 2, 2, 4, 6], dtype=torch.int64) if with_csr else None,
        csr_col=torch.tensor([0, 1, 2, 3, 1, 2], dtype=torch.int16) if with_csr else None,
        n_pat=2, nnz_pat=2, nnz=6)


@pytest.mark.parametrize("with_csr", [True, False])
def test_blocklist_round_trip(tmp_path, with_csr):
    bl = _cpu_blocklist(with_csr)
    p = tmp_path / "bl.npz"
    cba.save_blocklist(p, bl, layer=7)
    got, meta = cba.load_blocklist(p)
    assert meta["layer"] == 7
    for k in ("n_maps", "n_q_blocks", "n_k_blocks", "block_q", "block_k", "n_pat", "nnz_pat", "nnz"):
        assert getattr(got, k) == getattr(bl, k)
    for k in ("row_base", "row_pat", "pat_ptr", "pat_off", "csr_row_ptr", "csr_col"):
        a, b = getattr(got, k), getattr(bl, k)
        assert (a is None and b is None) or torch.equal(a, b)


def test_blocklist_sizes_are_checked(tmp_path):
    bl = _cpu_blocklist(True)
    bl.row_pat = bl.row_pat[:3]          # one row short of n_maps * n_q_blocks
    p = tmp_path / "bl.npz"
    cba.save_blocklist(p, bl)
    with pytest.raises(ValueError, match="row_pat has shape"):
        cba.load_blocklist(p)


def test_calibrate_resume_arguments():
    q = torch.zeros(2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="inputs_before"):
        cba.calibrate([q], [q], 250, inputs_before=4)
    with pytest.raises(ValueError, match="inputs_before"):
        cba.calibrate([q], [q], 250, inputs_before=-1)
