"""Test-side helpers: layout conversion of the GPU outputs for comparison with
the oracle. Written from the layout stated in include/qfp4.h, independently of
the library's own index function (which a test checks against this one)."""
from __future__ import annotations

import os
import tempfile

import numpy as np
import torch

# Scratch space of the tests that compile C helpers (kept inside the
# repository, git-ignored).
SCRATCH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_scratch")


def scratch_dir(prefix: str) -> str:
    """A fresh directory under the tests' scratch space."""
    os.makedirs(SCRATCH, exist_ok=True)
    return tempfile.mkdtemp(prefix=prefix, dir=SCRATCH)


def atom_offset(rows: int, kb: int, r, c):
    """Byte offset of scale (r, c) in the 512-byte-atom layout: atoms of 128
    rows x 4 scale columns, K-fastest; inside an atom byte (r%32)*16 +
    ((r//32)%4)*4 + c%4."""
    kb4 = (kb + 3) // 4 * 4
    return ((r // 128) * (kb4 // 4) + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)


def unswizzle_scales(flat: np.ndarray, rows: int, k: int, block: int) -> np.ndarray:
    """GPU scale buffer -> canonical [rows, k/block] codes."""
    kb = k // block
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    return flat[atom_offset(rows, kb, r, c)]


def padding_is_zero(flat: np.ndarray, rows: int, k: int, block: int) -> bool:
    """Every scale byte of the padded atoms outside [rows, k/block] is zero."""
    kb = k // block
    rows_p = (rows + 127) // 128 * 128
    kb4 = (kb + 3) // 4 * 4
    r = np.arange(rows_p)[:, None]
    c = np.arange(kb4)[None, :]
    off = atom_offset(rows, kb, r, c)
    pad = (r >= rows) | (c >= kb)
    return bool(np.all(flat[off[pad]] == 0))


def to_numpy_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.uint8)
