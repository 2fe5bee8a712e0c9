"""The C-ABI library without a GPU: it loads, exports every function
include/qfp4.h declares, and its host-only functions (sizes, the scale layout,
presets, error strings) behave as the header states."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from fp4_precision_b200 import qfp4 as Q

import helpers

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "qfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qfp4_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from fp4_precision_b200 import build
    build.build()
    return Q.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in Q._SIGNATURES, f"binding lacks {n}"


def test_strerror(lib):
    for s in (Q.OK, Q.ERR_INVALID_ARG, Q.ERR_MISALIGNED, Q.ERR_UNSUPPORTED_ARCH, Q.ERR_WORKSPACE, Q.ERR_CUDA,
              Q.ERR_TIMEOUT):
        assert lib.qfp4_strerror(s)
    assert lib.qfp4_strerror(12345) == b"unknown status"


@pytest.mark.parametrize("fmt", [Q.NVFP4, Q.MXFP4, Q.MXFP4_RU])
@pytest.mark.parametrize("rows,k", [(1, 64), (128, 128), (300, 320), (512, 4096), (129, 96)])
def test_scale_layout(lib, fmt, rows, k):
    nb = Q.BLOCK[fmt]
    if k % nb:
        pytest.skip("k not a multiple of the block")
    kb = k // nb
    nbytes = Q.scales_bytes(fmt, rows, k)
    assert nbytes == ((rows + 127) // 128) * ((kb + 3) // 4) * 512
    rows_p = (rows + 127) // 128 * 128
    kb4 = (kb + 3) // 4 * 4
    seen = np.zeros(nbytes, dtype=np.int32)
    for r in range(0, rows_p, max(1, rows_p // 97)):
        for c in range(kb4):
            off = Q.scale_offset(fmt, rows, k, r, c)
            assert off == helpers.atom_offset(rows, kb, r, c)
            seen[off] += 1
    full = np.zeros(nbytes, dtype=np.int32)
    r = np.arange(rows_p)[:, None]
    c = np.arange(kb4)[None, :]
    np.add.at(full, helpers.atom_offset(rows, kb, r, c).ravel(), 1)
    assert np.all(full == 1), "the layout is a bijection onto the buffer"
    assert Q.scale_offset(fmt, rows, k, rows_p, 0) == -1 and Q.scale_offset(fmt, rows, k, 0, kb4) == -1


def test_sizes(lib):
    assert Q.codes_bytes(10, 64) == 320
    assert Q.codes_bytes(0, 64) == 0
    assert Q.scales_bytes(7, 10, 64) == 0
    assert Q.scales_bytes(Q.MXFP4_RU, 128, 256) == Q.scales_bytes(Q.MXFP4, 128, 256)
    assert Q.quantize_workspace_bytes() >= 4 * 148


@pytest.mark.parametrize("name", ["NVIDIA_NVFP4", "QUARTET2_NVFP4", "AMD_MXFP4_H"])
def test_presets_match_oracle(lib, name):
    r = Q.recipe(name)
    o = O.preset(name)
    for g, og in ((r.fprop, o.fprop), (r.dgrad, o.dgrad), (r.wgrad, o.wgrad)):
        assert (g.fmt, g.rnd_a, g.rnd_b, g.had) == (og.fmt, og.rnd_a, og.rnd_b, og.had)
    bad = Q.Recipe()
    assert lib.qfp4_recipe_preset(99, ctypes.byref(bad)) == Q.ERR_INVALID_ARG


def test_linear_workspace_covers_operands(lib):
    r = Q.recipe("QUARTET2_NVFP4")
    M, N, K = 1024, 768, 512
    fwd = Q.linear_workspace_bytes(False, M, N, K, r)
    bwd = Q.linear_workspace_bytes(True, M, N, K, r)
    assert fwd >= Q.codes_bytes(M, K) + Q.codes_bytes(N, K) + Q.scales_bytes(0, M, K) + Q.scales_bytes(0, N, K)
    assert bwd >= (Q.codes_bytes(M, N) + Q.codes_bytes(K, N) + Q.codes_bytes(N, M) + Q.codes_bytes(K, M))


def test_launch_counter(lib):
    Q.launch_count(reset=True)
    assert Q.launch_count() == 0


def test_binding_has_no_fallback(lib, monkeypatch):
    """Without the built library the binding raises instead of computing
    anything itself, and on a host without a GPU a quantization raises too
    (no CPU path exists to fall back to)."""
    import torch
    monkeypatch.setattr(Q, "_lib", None)
    monkeypatch.setattr(Q, "LIB_PATH", os.path.join(ROOT, "fp4_precision_b200", "no_such_libqfp4.so"))
    with pytest.raises(RuntimeError, match="missing"):
        Q.lib()
    monkeypatch.undo()
    if not torch.cuda.is_available():
        x = torch.zeros((128, 128), dtype=torch.bfloat16)
        with pytest.raises(Exception):
            Q.quantize(x, Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW)

