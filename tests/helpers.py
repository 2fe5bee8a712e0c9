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


# ---------------------------------------------------------------------------
# Canary guard bytes around GPU output buffers (out-of-bounds write evidence)

GUARD_BYTES = 4096    # a multiple of 16 and of 128: the view keeps the alignment TMA stores need
GUARD_PATTERN = 0xA5


class Guarded:
    """A device buffer of `nbytes` between two guard regions of GUARD_BYTES
    filled with GUARD_PATTERN; `view(dtype, shape)` is the usable middle."""

    def __init__(self, nbytes: int, device):
        self.nbytes = int(nbytes)
        self.base = torch.full((self.nbytes + 2 * GUARD_BYTES,), GUARD_PATTERN, dtype=torch.uint8, device=device)

    def view(self, dtype, shape):
        mid = self.base[GUARD_BYTES:GUARD_BYTES + self.nbytes]
        return mid.view(dtype).view(shape)

    def intact(self) -> bool:
        g = self.base.cpu().numpy()
        return bool(np.all(g[:GUARD_BYTES] == GUARD_PATTERN) and np.all(g[GUARD_BYTES + self.nbytes:] == GUARD_PATTERN))


def guarded_qtensor(Q, fmt: int, rows: int, k: int, device):
    """A quantized-operand buffer (codes, scales, tensor scale) whose three
    parts each sit between guard bytes; returns (qtensor, guards)."""
    gc = Guarded(max(rows * k // 2, 16), device)
    gs = Guarded(max(Q.scales_bytes(fmt, rows, k), 16), device)
    gt = Guarded(16, device)
    codes = gc.view(torch.uint8, (max(rows * k // 2, 16),))[: rows * k // 2].view(rows, k // 2)
    scales = gs.view(torch.uint8, (gs.nbytes,))
    ts = gt.view(torch.float32, (4,))[:1]
    desc = Q.TensorDesc(codes.data_ptr(), scales.data_ptr(), ts.data_ptr(), 0, 0, 0, 0, 0, 0, 0)
    return Q.QTensor(codes, scales, ts, desc), (gc, gs, gt)


def guarded_matrix(rows: int, cols: int, dtype, device):
    """A [rows, cols] output matrix between guard bytes; returns (tensor, guard)."""
    esz = torch.tensor([], dtype=dtype).element_size()
    g = Guarded(max(rows * cols * esz, 16), device)
    return g.view(torch.uint8, (g.nbytes,))[: rows * cols * esz].view(dtype).view(rows, cols), g


def assert_guards_intact(*guards):
    torch.cuda.synchronize()
    for g in guards:
        if isinstance(g, (tuple, list)):
            assert_guards_intact(*g)
        else:
            assert g.intact(), "a kernel wrote outside its output buffer (canary bytes changed)"
