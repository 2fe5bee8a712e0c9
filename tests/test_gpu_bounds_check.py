"""The bounds-checked build (libqfp4_bc.so, QFP4_BOUNDS_CHECK): every kernel
store address is checked against the buffer its arguments describe, and a
store outside is dropped and reported by qfp4_status as QFP4_ERR_BOUNDS. A
child process runs the library's entry points with that build on ragged
shapes (partial tiles on both axes, both GEMM kernels, every output kind) and
checks the status after each call; the parent runs the same calls with the
normal build and requires byte-identical outputs."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import helpers

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def run_cases(Q, dev):
    """Every output of a fixed set of calls, as named uint8 arrays (status
    checked after each call)."""
    out = {}
    g = torch.Generator(device="cpu").manual_seed(7)

    def rnd(*shape):
        return (torch.randn(shape, generator=g) * torch.rand(shape[-1], generator=g) * 3).to(torch.bfloat16).to(dev)

    def keep(name, *ts):
        Q.status()
        for i, t in enumerate(ts):
            out[f"{name}.{i}"] = t.detach().contiguous().view(torch.uint8).cpu().numpy().ravel()

    seed = Q.make_seed(11, 12, 3, 4)
    x = rnd(352, 416)
    for fmt in (Q.NVFP4, Q.MXFP4, Q.MXFP4_RU):
        for rnd_mode in (Q.RTN, Q.SR, Q.QUARTET2):
            for had in (Q.HAD_NONE, Q.HAD_RAND16, Q.HAD_DET32):
                for axis in (Q.ROW, Q.COL):
                    q = Q.quantize(x, fmt, rnd_mode, had, axis, seed)
                    keep(f"q{fmt}{rnd_mode}{had}{axis}", q.codes, q.scales, q.tensor_scale)
    xb = rnd(320, 448)  # the column kernel over 64-row bands (R a multiple of 64), ragged columns
    for rnd_mode in (Q.RTN, Q.QUARTET2):
        q = Q.quantize(xb, Q.NVFP4, rnd_mode, Q.HAD_RAND16, Q.COL, seed)
        keep(f"band{rnd_mode}", q.codes, q.scales)
        s_col = Q.make_seed(5, 6, 1, 2)
        am_row, am_col = Q.amax(xb, Q.HAD_RAND16, Q.ROW, seed), Q.amax(xb, Q.HAD_RAND16, Q.COL, s_col)
        qr, qc = Q.quantize_dual(xb, Q.NVFP4, rnd_mode, Q.HAD_RAND16, Q.HAD_RAND16, seed, s_col, am_row, am_col)
        keep(f"dual{rnd_mode}", qr.codes, qr.scales, qc.codes, qc.scales)
    keep("amax", Q.amax(x, Q.HAD_RAND16, Q.COL, seed))
    keep("amax_rowcol", Q.amax_rowcol(xb, Q.HAD_RAND16, seed, Q.make_seed(5, 6, 1, 2)))
    # single-CTA kernel (M <= 128) and CTA pairs; N ragged against the 256-wide
    # tiles (the quantizing epilogue needs N a multiple of 32, the amax one of 16)
    for M, K, N, Nq, Na in ((100, 192, 200, 224, 208), (300, 448, 328, 352, 336)):
        A = Q.quantize(rnd(M, K), Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW, seed)
        B = Q.quantize(rnd(N, K), Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW, seed)
        keep(f"gemm_bf16_{M}", Q.gemm(A, B, torch.bfloat16))
        keep(f"gemm_f32_{M}", Q.gemm(A, B, torch.float32))
        acc = torch.ones((M, N), dtype=torch.float32, device=dev)
        keep(f"gemm_acc_{M}", Q.gemm_accumulate(A, B, acc))
        Am = Q.quantize(rnd(M, K), Q.MXFP4, Q.RTN, Q.HAD_NONE, Q.ROW, seed)
        Bm = Q.quantize(rnd(Nq, K), Q.MXFP4, Q.RTN, Q.HAD_NONE, Q.ROW, seed)
        D, qo = Q.gemm_quantize(Am, Bm, Q.HAD_DET32, seed)
        keep(f"gemm_q_{M}", D, qo.codes, qo.scales)
        Ba = Q.quantize(rnd(Na, K), Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW, seed)
        D, am = Q.gemm_amax(A, Ba, Q.HAD_RAND16, seed)
        keep(f"gemm_amax_{M}", D, am)
    # the linear layer takes M, N, K multiples of 128: 384 and 640 leave half tiles
    X, W, dY = rnd(384, 640), rnd(384, 640), rnd(384, 384)
    for name in ("QUARTET2_NVFP4", "NVIDIA_NVFP4", "AMD_MXFP4_H"):
        rec = Q.recipe(name)
        keep(f"fwd_{name}", Q.linear_fwd(X, W, rec, seed))
        keep(f"bwd_{name}", *Q.linear_bwd(dY, X, W, rec, seed))
    return out


CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
from fp4_precision_b200 import qfp4 as Q
assert Q.LIB_PATH.endswith("libqfp4_bc.so"), Q.LIB_PATH
import test_gpu_bounds_check as T
np.savez({out!r}, **T.run_cases(Q, torch.device("cuda", 0)))
"""


def test_bounds_checked_build_matches_and_stays_in_bounds():
    from fp4_precision_b200 import qfp4 as Q
    from fp4_precision_b200 import build
    build.build(bounds_check=True)  # no-op when the in-tree library is up to date
    d = helpers.scratch_dir("bounds_")
    path = os.path.join(d, "bc.npz")
    env = dict(os.environ, QFP4_BOUNDS_CHECK="1")
    subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), out=path)],
                   env=env, check=True, timeout=900)
    checked = np.load(path)
    plain = run_cases(Q, torch.device("cuda", 0))
    assert sorted(checked.files) == sorted(plain)
    for k, v in plain.items():
        assert np.array_equal(checked[k], v), k
