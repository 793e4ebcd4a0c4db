"""O5 -- compile block masks into per-row kept-block lists.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

CalibAtt compiles the calibrated patterns into attention operations for each
layer, head and diffusion timestep (paper page, Abstract), and within-frame
patterns repeat across spatial rows (Figure 4(b)).  Reading taken for the
storage: rows are scanned in (map, query block) order, map id =
(layer * T + timestep) * H + head.  Each row's kept key blocks are listed in
ascending order; a row is stored as its base (first kept block, 0 for an empty
row) plus the offsets ``kb - base``.  Identical offset lists -- rows that are
translates of one another -- are stored once in a pattern pool, numbered in
order of first occurrence; pattern 0 is the empty pattern and always exists.
With ``dedup=False`` every non-empty row gets a pattern of its own.  A plain
CSR (row pointers and columns) is produced as well.
"""

from __future__ import annotations

import numpy as np


def compile_blocklist(masks, dedup=True):
    """``masks``: [n_maps, nqb, nkb] 0/1.  Returns a dict of numpy arrays."""
    masks = np.asarray(masks)
    n_maps, nqb, nkb = masks.shape
    rows = masks.reshape(n_maps * nqb, nkb)
    n_rows = rows.shape[0]
    row_base = np.zeros(n_rows, dtype=np.int32)
    row_pat = np.zeros(n_rows, dtype=np.int32)
    csr_row_ptr = np.zeros(n_rows + 1, dtype=np.int64)
    cols_all = []
    pool = {}                 # offsets bytes -> pattern id
    pat_lists = [np.zeros(0, dtype=np.int16)]
    for r in range(n_rows):
        cols = np.nonzero(rows[r])[0]
        csr_row_ptr[r + 1] = csr_row_ptr[r] + cols.size
        cols_all.append(cols.astype(np.int16))
        if cols.size == 0:
            row_base[r] = 0
            row_pat[r] = 0
            continue
        base = int(cols[0])
        offs = (cols - base).astype(np.int16)
        row_base[r] = base
        key = offs.tobytes()
        if dedup and key in pool:
            row_pat[r] = pool[key]
        else:
            pid = len(pat_lists)
            pat_lists.append(offs)
            if dedup:
                pool[key] = pid
            row_pat[r] = pid
    pat_ptr = np.zeros(len(pat_lists) + 1, dtype=np.int32)
    for i, lst in enumerate(pat_lists):
        pat_ptr[i + 1] = pat_ptr[i] + lst.size
    pat_off = np.concatenate(pat_lists).astype(np.int16) if pat_ptr[-1] else np.zeros(0, np.int16)
    csr_col = np.concatenate(cols_all).astype(np.int16) if csr_row_ptr[-1] else np.zeros(0, np.int16)
    return {
        "n_maps": n_maps, "n_q_blocks": nqb, "n_k_blocks": nkb,
        "row_base": row_base, "row_pat": row_pat,
        "pat_ptr": pat_ptr, "pat_off": pat_off,
        "csr_row_ptr": csr_row_ptr, "csr_col": csr_col,
        "n_pat": len(pat_lists), "nnz_pat": int(pat_ptr[-1]), "nnz": int(csr_row_ptr[-1]),
    }


def expand_blocklist(bl):
    """Inverse of ``compile_blocklist`` through the pattern pool: masks [n_maps, nqb, nkb]."""
    n_maps, nqb, nkb = bl["n_maps"], bl["n_q_blocks"], bl["n_k_blocks"]
    out = np.zeros((n_maps * nqb, nkb), dtype=np.uint8)
    ptr = np.asarray(bl["pat_ptr"])
    off = np.asarray(bl["pat_off"])
    for r in range(n_maps * nqb):
        p = int(bl["row_pat"][r])
        cols = int(bl["row_base"][r]) + off[ptr[p]:ptr[p + 1]].astype(np.int64)
        out[r, cols] = 1
    return out.reshape(n_maps, nqb, nkb)
