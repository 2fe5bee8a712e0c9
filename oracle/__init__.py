"""CPU oracle of the FP4 quantized-linear path (quantizers, GEMMs, linear layer).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package. The CUDA library never
does, and the two share no code: this package has its own C source
(``qfp4_oracle.c``), its own build step and its own constants.

The quantizer is plain C (fp32 decisions, see the C file's header); the
dequantization and the GEMMs are fp64 numpy, one library matmul per GEMM over
the dequantized operands, with no blocking or reordering.

Sources: the web pages "Quartet II - obuchenie v NVFP4 s tochnymi
nesmeshchyonnymi gradientami" (stuffynlp post 238), "New AMD paper overturns
conventional wisdom: FP4 training..." (sections "Chto takoe MXFP4",
"Poiskovaya eksperimental'naya rabota") and "NVIDIA sozdala metod obucheniya
neyrosetey v 4-bit tochnosti" (section "Kak eto rabotaet").
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qfp4_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lib = None

NVFP4, MXFP4, MXFP4_RU = 0, 1, 2
RTN, SR, QUARTET2 = 0, 1, 2
HAD_NONE, HAD_DET16, HAD_DET32, HAD_RAND16, HAD_RAND32 = 0, 1, 2, 3, 4
ROW, COL = 0, 1
TAG_ELEMENT, TAG_SCALE, TAG_SIGN = 0, 1, 2

BLOCK = {NVFP4: 16, MXFP4: 32, MXFP4_RU: 32}
HAD_N = {HAD_NONE: 0, HAD_DET16: 16, HAD_DET32: 32, HAD_RAND16: 16, HAD_RAND32: 32}

# Error bound of a GEMM output against the fp64 oracle, relative to sum_k |a_k b_k|.
GEMM_REL_BOUND = 2.0 ** -18


def compile_source(src: str, out: str) -> str:
    """gcc the oracle's C source (or a copy of it) into a shared library."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
         "-fno-fast-math", "-Wall", "-Wextra", "-Wno-unused-parameter", src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle's C source into ``oracle/_build/liboracle.so``."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


@contextlib.contextmanager
def using(path: str):
    """Run the oracle's Python layer on another build of the C source (the
    mutation tests use it to plant a mistake in a copy of the oracle)."""
    global _lib, _E2M1_TABLE
    saved = _lib, _E2M1_TABLE
    _lib, _E2M1_TABLE = load(path), None
    try:
        yield
    finally:
        _lib, _E2M1_TABLE = saved


def load(path: str) -> ctypes.CDLL:
    """Load a build of the oracle's C source and declare its signatures."""
    L = ctypes.CDLL(path)
    u8, u32, u64, i64, f32p = ctypes.c_uint8, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
    L.oracle_philox4x32_10.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    L.oracle_random_word.argtypes = [u64, u32, u32, u64]
    L.oracle_random_word.restype = u32
    L.oracle_element_uniform.argtypes = [u64, u32, u64]
    L.oracle_element_uniform.restype = ctypes.c_float
    L.oracle_e2m1_value.argtypes = [u8]
    L.oracle_e2m1_value.restype = ctypes.c_double
    L.oracle_e2m1_rtn.argtypes = [ctypes.c_float]
    L.oracle_e2m1_rtn.restype = u8
    L.oracle_e2m1_sr.argtypes = [ctypes.c_float, ctypes.c_float]
    L.oracle_e2m1_sr.restype = u8
    L.oracle_e4m3_value.argtypes = [u8]
    L.oracle_e4m3_value.restype = ctypes.c_double
    L.oracle_e4m3_rne_sat.argtypes = [ctypes.c_float]
    L.oracle_e4m3_rne_sat.restype = u8
    L.oracle_e4m3_sr.argtypes = [ctypes.c_float, ctypes.c_float]
    L.oracle_e4m3_sr.restype = u8
    L.oracle_e8m0_value.argtypes = [u8]
    L.oracle_e8m0_value.restype = ctypes.c_double
    L.oracle_e8m0_sr.argtypes = [ctypes.c_float, ctypes.c_float]
    L.oracle_e8m0_sr.restype = u8
    L.oracle_hadamard_matrix.argtypes = [ctypes.c_int, ctypes.c_void_p]
    L.oracle_fwht.argtypes = [ctypes.c_void_p, ctypes.c_int]
    L.oracle_sign_bits.argtypes = [u64, u32]
    L.oracle_sign_bits.restype = u32
    L.oracle_quantize.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, u64, u32, u64, u32, f32p, ctypes.c_void_p, ctypes.c_void_p,
                                  f32p, f32p]
    L.oracle_quantize.restype = ctypes.c_int
    L.oracle_quantize_rows.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, u64, u32, u64, u32, f32p, ctypes.c_void_p, i64,
                                       ctypes.c_void_p, ctypes.c_void_p, f32p, f32p]
    L.oracle_quantize_rows.restype = ctypes.c_int
    L.oracle_rotate.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_int, ctypes.c_int, u64, u32,
                                ctypes.c_void_p]
    L.oracle_rotate.restype = ctypes.c_int
    return L


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


# ---------------------------------------------------------------------------
# scalar helpers (thin wrappers over the C functions)

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    lib().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def random_word(seed: int, tag: int, stream: int, i: int) -> int:
    return int(lib().oracle_random_word(seed, tag, stream, i))


def element_uniform(seed: int, stream: int, i: int) -> float:
    """The uniform of element i's stochastic rounding (16 bits, two per word)."""
    return float(lib().oracle_element_uniform(seed, stream, i))


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(code)


def e2m1_rtn(u: float) -> int:
    return lib().oracle_e2m1_rtn(u)


def e2m1_sr(u: float, rho: float) -> int:
    return lib().oracle_e2m1_sr(u, rho)


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(code)


def e4m3_rne_sat(t: float) -> int:
    return lib().oracle_e4m3_rne_sat(t)


def e4m3_sr(t: float, rho: float) -> int:
    return lib().oracle_e4m3_sr(t, rho)


def e8m0_value(code: int) -> float:
    return lib().oracle_e8m0_value(code)


def e8m0_sr(t: float, rho: float) -> int:
    """Stochastic rounding of t > 0 onto powers of two: the E8M0 code."""
    return lib().oracle_e8m0_sr(t, rho)


def hadamard_matrix(n: int) -> np.ndarray:
    H = np.zeros((n, n), dtype=np.int8)
    lib().oracle_hadamard_matrix(n, _ptr(H))
    return H


def fwht(w: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(np.array(w, dtype=np.float32))
    lib().oracle_fwht(_ptr(v), v.size)
    return v


def sign_bits(rot_seed: int, rot_stream: int = 0) -> int:
    return int(lib().oracle_sign_bits(rot_seed, rot_stream))


# ---------------------------------------------------------------------------
# tensors

def _as_bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor (CPU) or a uint16 numpy array of bf16 bits."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


@dataclass
class QTensor:
    """Quantized tensor in the quantized orientation: rows x k, k the reduction axis."""
    codes: np.ndarray      # uint8 [rows, k/2], element j of a row in nibble j%2 of byte j/2 (low first)
    scales: np.ndarray     # uint8 [rows, k/nb], canonical row-major scale codes
    g: float               # NVFP4 per-tensor scale (1.0 for MXFP4)
    fmt: int
    had: int
    rows: int
    k: int
    alpha: np.ndarray | None = None  # Quartet II renormalisation per block (1.0 otherwise)


def quantize(x, fmt: int, rnd: int, had: int, axis: int, rot_seed: int = 0, rot_stream: int = 0,
             sr_seed: int = 0, sr_stream: int = 0, amax: float | None = None, rows_sel=None) -> QTensor:
    """Quantize x (bf16 [R, C]). rows_sel (optional): only these rows of the
    quantized orientation, in that order (the tensor amax and the random words
    stay those of the whole tensor); the result then has len(rows_sel) rows."""
    xb = _as_bf16_bits(x)
    R, C = xb.shape
    rows, k = (R, C) if axis == ROW else (C, R)
    nb = BLOCK[fmt]
    sel = None if rows_sel is None else np.ascontiguousarray(np.asarray(rows_sel, dtype=np.int64))
    n_out = rows if sel is None else len(sel)
    codes = np.zeros((n_out, k // 2), dtype=np.uint8)
    scales = np.zeros((n_out, k // nb), dtype=np.uint8)
    alpha = np.ones((n_out, k // nb), dtype=np.float32)
    g = np.zeros(1, dtype=np.float32)
    am = None if amax is None else np.array([amax], dtype=np.float32)
    rc = lib().oracle_quantize_rows(_ptr(xb), R, C, C, fmt, rnd, had, axis, rot_seed, rot_stream, sr_seed,
                                    sr_stream, None if am is None else _ptr(am),
                                    None if sel is None else _ptr(sel), 0 if sel is None else len(sel),
                                    _ptr(codes), _ptr(scales), _ptr(g), _ptr(alpha))
    if rc != 0:
        raise ValueError("oracle_quantize: invalid arguments")
    return QTensor(codes, scales, float(g[0]), fmt, had, n_out, k, alpha)


def rotate(x, had: int, axis: int, rot_seed: int = 0, rot_stream: int = 0) -> np.ndarray:
    xb = _as_bf16_bits(x)
    R, C = xb.shape
    rows, k = (R, C) if axis == ROW else (C, R)
    v = np.zeros((rows, k), dtype=np.float32)
    if lib().oracle_rotate(_ptr(xb), R, C, C, had, axis, rot_seed, rot_stream, _ptr(v)) != 0:
        raise ValueError("oracle_rotate: invalid arguments")
    return v


_E2M1_TABLE = None


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """uint8 [rows, k/2] -> uint8 [rows, k] of 4-bit codes (low nibble first)."""
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = codes & 0x0F
    out[:, 1::2] = codes >> 4
    return out


def scale_values(q: QTensor) -> np.ndarray:
    """fp64 value of each block scale, [rows, k/nb]."""
    decode = e4m3_value if q.fmt == NVFP4 else e8m0_value
    table = np.array([decode(c) for c in range(256)], dtype=np.float64)
    return table[q.scales]


def dequantize(q: QTensor) -> np.ndarray:
    """x_hat = q * S * g (NVFP4) or q * 2^E (MXFP4), fp64, in the rotated domain.
    Every product is exact in fp64 (<= 3 + 4 + 24 significant bits)."""
    global _E2M1_TABLE
    if _E2M1_TABLE is None:
        _E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
    vals = _E2M1_TABLE[unpack_codes(q.codes)]
    nb = BLOCK[q.fmt]
    s = np.repeat(scale_values(q), nb, axis=1)
    out = vals * s
    if q.fmt == NVFP4:
        out = out * np.float64(q.g)
    return out


def unrotate(xhat: np.ndarray, had: int, rot_seed: int = 0, rot_stream: int = 0) -> np.ndarray:
    """Map a rotated-domain estimate back: per n_h chunk, D H x_hat / sqrt(n_h), fp64."""
    nh = HAD_N[had]
    if nh == 0:
        return xhat.copy()
    H = hadamard_matrix(nh).astype(np.float64)
    bits = sign_bits(rot_seed, rot_stream) if had in (HAD_RAND16, HAD_RAND32) else 0
    d = np.array([-1.0 if (bits >> j) & 1 else 1.0 for j in range(nh)])
    rows, k = xhat.shape
    chunks = xhat.reshape(rows, k // nh, nh)
    out = (chunks @ H.T) / np.sqrt(nh) * d
    return out.reshape(rows, k)


def gemm(A: QTensor, B: QTensor) -> np.ndarray:
    """D = A_hat . B_hat^T in fp64 over the dequantized operands (both rotated the
    same way, so the rotation cancels). [AMD MXFP4] "Poiskovaya...": the three
    GEMMs of a linear layer are products of this form."""
    assert A.k == B.k
    return dequantize(A) @ dequantize(B).T


def gemm_bound(A: QTensor, B: QTensor) -> np.ndarray:
    """Per-output tolerance 2^-18 * sum_k |a_k b_k|."""
    return GEMM_REL_BOUND * (np.abs(dequantize(A)) @ np.abs(dequantize(B)).T)


# ---------------------------------------------------------------------------
# linear layer: which operand gets which quantization ([AMD MXFP4]
# "Poiskovaya...": Fprop Y = X W^T, Dgrad dX = dY W, Wgrad dW = dY^T X)

@dataclass
class GemmCfg:
    fmt: int
    rnd_a: int
    rnd_b: int
    had: int


@dataclass
class Recipe:
    fprop: GemmCfg
    dgrad: GemmCfg
    wgrad: GemmCfg


def preset(name: str) -> Recipe:
    """The recipes the pages describe.
    NVIDIA_NVFP4: [NVIDIA NVFP4] "Kak eto rabotaet" - 16x16 random Hadamard on the
      weight-gradient inputs, stochastic rounding of the gradient.
    QUARTET2_NVFP4: [Quartet II] - RTN forward (its "more precise forward" is not
      specified on the page), random rotation + Quartet II scale SR backward.
    AMD_MXFP4_H: [AMD MXFP4] - MXFP4 everywhere, deterministic Hadamard on Wgrad.
    """
    if name == "NVIDIA_NVFP4":
        return Recipe(GemmCfg(NVFP4, RTN, RTN, HAD_NONE), GemmCfg(NVFP4, SR, RTN, HAD_NONE),
                      GemmCfg(NVFP4, SR, RTN, HAD_RAND16))
    if name == "QUARTET2_NVFP4":
        return Recipe(GemmCfg(NVFP4, RTN, RTN, HAD_DET16), GemmCfg(NVFP4, QUARTET2, QUARTET2, HAD_RAND16),
                      GemmCfg(NVFP4, QUARTET2, QUARTET2, HAD_RAND16))
    if name == "AMD_MXFP4_H":
        return Recipe(GemmCfg(MXFP4, RTN, RTN, HAD_NONE), GemmCfg(MXFP4, RTN, RTN, HAD_NONE),
                      GemmCfg(MXFP4, RTN, RTN, HAD_DET32))
    raise KeyError(name)


# Stream ids of the linear layer: the rotation stream is the GEMM (0 Fprop,
# 1 Dgrad, 2 Wgrad), shared by both operands; the rounding stream is the operand.
GEMM_FPROP, GEMM_DGRAD, GEMM_WGRAD = 0, 1, 2
OP_X_FPROP, OP_W_FPROP, OP_DY_DGRAD, OP_W_DGRAD, OP_DY_WGRAD, OP_X_WGRAD = 0, 1, 2, 3, 4, 5


def linear_fwd_operands(X, W, recipe: Recipe, rot_seed: int, sr_seed: int):
    c = recipe.fprop
    A = quantize(X, c.fmt, c.rnd_a, c.had, ROW, rot_seed, GEMM_FPROP, sr_seed, OP_X_FPROP)
    B = quantize(W, c.fmt, c.rnd_b, c.had, ROW, rot_seed, GEMM_FPROP, sr_seed, OP_W_FPROP)
    return A, B


def linear_bwd_operands(dY, X, W, recipe: Recipe, rot_seed: int, sr_seed: int):
    d, w = recipe.dgrad, recipe.wgrad
    # Dgrad dX[M,K] = dY[M,N] W[N,K]: reduce over N. A = dY along N (row),
    # B = W along N (col, i.e. the quantized W^T [K, N]).
    Ad = quantize(dY, d.fmt, d.rnd_a, d.had, ROW, rot_seed, GEMM_DGRAD, sr_seed, OP_DY_DGRAD)
    Bd = quantize(W, d.fmt, d.rnd_b, d.had, COL, rot_seed, GEMM_DGRAD, sr_seed, OP_W_DGRAD)
    # Wgrad dW[N,K] = dY^T[N,M] X[M,K]: reduce over M (tokens). A = dY along M
    # (col -> dY^T [N, M]), B = X along M (col -> X^T [K, M]).
    Aw = quantize(dY, w.fmt, w.rnd_a, w.had, COL, rot_seed, GEMM_WGRAD, sr_seed, OP_DY_WGRAD)
    Bw = quantize(X, w.fmt, w.rnd_b, w.had, COL, rot_seed, GEMM_WGRAD, sr_seed, OP_X_WGRAD)
    return Ad, Bd, Aw, Bw


def linear_fwd(X, W, recipe: Recipe, rot_seed: int = 0, sr_seed: int = 0):
    A, B = linear_fwd_operands(X, W, recipe, rot_seed, sr_seed)
    return gemm(A, B), gemm_bound(A, B)


def linear_bwd(dY, X, W, recipe: Recipe, rot_seed: int = 0, sr_seed: int = 0):
    Ad, Bd, Aw, Bw = linear_bwd_operands(dY, X, W, recipe, rot_seed, sr_seed)
    return (gemm(Ad, Bd), gemm_bound(Ad, Bd)), (gemm(Aw, Bw), gemm_bound(Aw, Bw))
