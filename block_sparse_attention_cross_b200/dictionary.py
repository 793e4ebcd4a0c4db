"""Saving and loading the offline products of calibration.

Calibration produces plain arrays (paper page, Figure 3(b): how often each
key block was kept across the calibration prompts; Figure 5(a): the
per-(layer, timestep, head) mask dictionary; Abstract: the compiled kept-block
lists).  They are written as one ``.npz`` archive holding the arrays and a
JSON header: the format tag, the caller's metadata (block sizes, rho, the
selection rule, ...), and per array its shape, dtype and SHA-256.  Reading
checks every array against the header, so a truncated or altered file is
refused instead of silently producing a different mask.

Vote counts and energy sums add up over inputs, so a calibration saved after
n inputs resumes at input n + 1: load the state and pass ``votes``,
``energy_sum`` and ``inputs_before=n`` to :func:`calibrate`.

Host I/O only; nothing here computes any part of the method.
"""

from __future__ import annotations

import hashlib
import json

import numpy as np
import torch

FORMAT = "calibatt-state/1"
_HEADER = "__header__"
_DTYPES = ("uint8", "int16", "int32", "int64", "float32", "float64")


def _as_numpy(name, t):
    if isinstance(t, torch.Tensor):
        if t.dtype == torch.bfloat16:
            raise TypeError(f"{name}: bfloat16 arrays are not stored (no numpy dtype)")
        a = t.detach().cpu().contiguous().numpy()
    else:
        a = np.ascontiguousarray(t)
    if a.dtype.name not in _DTYPES:
        raise TypeError(f"{name}: dtype {a.dtype} is not one of {', '.join(_DTYPES)}")
    return a


def _digest(a):
    return hashlib.sha256(a.tobytes()).hexdigest()


def save_state(path, arrays, meta=None):
    """Writes ``arrays`` (name -> tensor or ndarray) and ``meta`` (a
    JSON-serialisable dict) to ``path`` as one ``.npz`` archive with a checked
    header.  Returns ``path``."""
    header = {"format": FORMAT, "meta": dict(meta or {}), "arrays": {}}
    payload = {}
    for name, t in arrays.items():
        if not name.isidentifier() or name.startswith("__"):
            raise ValueError(f"array name {name!r} must be an identifier not starting with '__'")
        a = _as_numpy(name, t)
        header["arrays"][name] = {"shape": list(a.shape), "dtype": a.dtype.name, "sha256": _digest(a)}
        payload[name] = a
    payload[_HEADER] = np.frombuffer(json.dumps(header, sort_keys=True).encode("utf-8"), dtype=np.uint8)
    with open(path, "wb") as f:
        np.savez(f, **payload)
    return path


def load_state(path, device=None):
    """Reads an archive written by :func:`save_state`.  Returns (arrays as
    torch tensors, on ``device`` when given, meta).  Raises ValueError when the
    format tag, the set of arrays, or any array's shape, dtype or SHA-256
    differs from the header."""
    with np.load(path, allow_pickle=False) as z:
        if _HEADER not in z.files:
            raise ValueError(f"{path}: no header")
        header = json.loads(bytes(z[_HEADER]).decode("utf-8"))
        if header.get("format") != FORMAT:
            raise ValueError(f"{path}: format {header.get('format')!r}, expected {FORMAT!r}")
        specs = header["arrays"]
        names = set(z.files) - {_HEADER}
        if names != set(specs):
            raise ValueError(f"{path}: arrays {sorted(names)} do not match the header's {sorted(specs)}")
        out = {}
        for name, spec in specs.items():
            a = z[name]
            if list(a.shape) != spec["shape"] or a.dtype.name != spec["dtype"]:
                raise ValueError(f"{path}: {name} is {a.dtype} {list(a.shape)}, header says "
                                 f"{spec['dtype']} {spec['shape']}")
            if _digest(a) != spec["sha256"]:
                raise ValueError(f"{path}: {name} does not match its SHA-256")
            t = torch.from_numpy(np.array(a))
            out[name] = t.to(device) if device is not None else t
    return out, header["meta"]


def save_calibration(path, votes, energy_sum, inputs_seen, **meta):
    """Calibration state after ``inputs_seen`` inputs: vote counts (int32) and
    energy sums (float32), both [H, nqb, nkb], plus the caller's parameters."""
    if tuple(votes.shape) != tuple(energy_sum.shape) or votes.dim() != 3:
        raise ValueError("votes and energy_sum must share one [H, nqb, nkb] shape")
    if votes.dtype != torch.int32 or energy_sum.dtype != torch.float32:
        raise ValueError("votes must be int32 and energy_sum float32")
    if int(inputs_seen) < 1:
        raise ValueError("inputs_seen must be >= 1")
    return save_state(path, {"votes": votes, "energy_sum": energy_sum},
                      dict(meta, kind="calibration", inputs_seen=int(inputs_seen)))


def load_calibration(path, device=None):
    """Returns (votes, energy_sum, inputs_seen, meta) saved by :func:`save_calibration`."""
    arrays, meta = load_state(path, device)
    if meta.get("kind") != "calibration":
        raise ValueError(f"{path}: not a calibration state")
    return arrays["votes"], arrays["energy_sum"], int(meta["inputs_seen"]), meta


def save_masks(path, masks, **meta):
    """A mask dictionary: uint8 [n_maps, nqb, nkb], map id = (l T + t) H + h."""
    if masks.dtype != torch.uint8 or masks.dim() != 3:
        raise ValueError("masks must be uint8 [n_maps, nqb, nkb]")
    return save_state(path, {"masks": masks}, dict(meta, kind="masks"))


def load_masks(path, device=None):
    """Returns (masks, meta) saved by :func:`save_masks`."""
    arrays, meta = load_state(path, device)
    if meta.get("kind") != "masks":
        raise ValueError(f"{path}: not a mask dictionary")
    return arrays["masks"], meta


_BL_INTS = ("n_maps", "n_q_blocks", "n_k_blocks", "block_q", "block_k", "n_pat", "nnz_pat", "nnz")
_BL_ARRAYS = ("row_base", "row_pat", "pat_ptr", "pat_off", "csr_row_ptr", "csr_col")


def save_blocklist(path, bl, **meta):
    """A compiled kept-block list (:class:`BlockList`), CSR included when present."""
    arrays = {k: getattr(bl, k) for k in _BL_ARRAYS if getattr(bl, k) is not None}
    sizes = {k: int(getattr(bl, k)) for k in _BL_INTS}
    return save_state(path, arrays, dict(meta, kind="blocklist", sizes=sizes))


def load_blocklist(path, device=None):
    """Returns (BlockList, meta) saved by :func:`save_blocklist`; the arrays
    are checked against the sizes they were compiled with."""
    from . import BlockList

    arrays, meta = load_state(path, device)
    if meta.get("kind") != "blocklist":
        raise ValueError(f"{path}: not a compiled block list")
    sz = meta["sizes"]
    rows = sz["n_maps"] * sz["n_q_blocks"]
    want = {"row_base": (rows,), "row_pat": (rows,), "pat_ptr": (sz["n_pat"] + 1,), "pat_off": (sz["nnz_pat"],),
            "csr_row_ptr": (rows + 1,), "csr_col": (sz["nnz"],)}
    for name, shape in want.items():
        if name in arrays and tuple(arrays[name].shape) != shape:
            raise ValueError(f"{path}: {name} has shape {tuple(arrays[name].shape)}, the sizes give {shape}")
    if ("csr_row_ptr" in arrays) != ("csr_col" in arrays):
        raise ValueError(f"{path}: csr_row_ptr and csr_col must be stored together")
    bl = BlockList(sz["n_maps"], sz["n_q_blocks"], sz["n_k_blocks"], sz["block_q"], sz["block_k"],
                   row_base=arrays["row_base"], row_pat=arrays["row_pat"], pat_ptr=arrays["pat_ptr"],
                   pat_off=arrays["pat_off"], csr_row_ptr=arrays.get("csr_row_ptr"), csr_col=arrays.get("csr_col"),
                   n_pat=sz["n_pat"], nnz_pat=sz["nnz_pat"], nnz=sz["nnz"])
    return bl, meta
