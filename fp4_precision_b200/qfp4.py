"""ctypes binding of the C ABI in include/qfp4.h (argument marshalling only).

Every step of the quantizers, GEMMs and linear layer runs in the sm_100a CUDA
library ``libqfp4.so`` built from ``csrc/``; PyTorch provides device memory
and streams. There is no fallback: if the library is missing or the device is
not a B200 the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QFP4_BOUNDS_CHECK=1 selects the bounds-checked build (libqfp4_bc.so): the
# same kernels with every store address checked, reported by qfp4_status
LIB_PATH = os.path.join(_HERE, "libqfp4_bc.so" if os.environ.get("QFP4_BOUNDS_CHECK") == "1" else "libqfp4.so")

NVFP4, MXFP4, MXFP4_RU = 0, 1, 2
RTN, SR, QUARTET2 = 0, 1, 2
HAD_NONE, HAD_DET16, HAD_DET32, HAD_RAND16, HAD_RAND32 = 0, 1, 2, 3, 4
ROW, COL = 0, 1
OUT_BF16, OUT_F32 = 0, 1
PRESETS = {"NVIDIA_NVFP4": 0, "QUARTET2_NVFP4": 1, "AMD_MXFP4_H": 2}
BLOCK = {NVFP4: 16, MXFP4: 32, MXFP4_RU: 32}

OK, ERR_INVALID_ARG, ERR_MISALIGNED, ERR_UNSUPPORTED_ARCH, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5, -6
ERR_TOO_LARGE = -7
ERR_BOUNDS = -8
NOALLOC_SCRATCH_BYTES = 32 << 20
ROUND_E2M1_SR, ROUND_E2M1_RN, ROUND_E4M3_SR, ROUND_E4M3_RN, ROUND_E8M0_SR = 0, 1, 2, 3, 4


class Seed(ctypes.Structure):
    _fields_ = [("rot", ctypes.c_uint64), ("sr", ctypes.c_uint64), ("rot_stream", ctypes.c_uint32),
                ("sr_stream", ctypes.c_uint32)]


class TensorDesc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("k", ctypes.c_int64), ("fmt", ctypes.c_int32), ("had", ctypes.c_int32),
                ("rot_seed", ctypes.c_uint64), ("rot_stream", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class GemmCfg(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("rnd_a", ctypes.c_int32), ("rnd_b", ctypes.c_int32), ("had", ctypes.c_int32)]


class Recipe(ctypes.Structure):
    _fields_ = [("fprop", GemmCfg), ("dgrad", GemmCfg), ("wgrad", GemmCfg), ("y_dtype", ctypes.c_int32),
                ("dx_dtype", ctypes.c_int32), ("dw_dtype", ctypes.c_int32), ("dw_accumulate", ctypes.c_int32)]


class QFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib().qfp4_strerror(status).decode()
        if status == ERR_CUDA:
            msg += f" (cudaError {lib().qfp4_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")
        self.status = status


_lib = None
_VOID, _I32, _I64, _U64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t

_SIGNATURES = {
    "qfp4_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "qfp4_last_cuda_error": (ctypes.c_int, []),
    "qfp4_codes_bytes": (_SZ, [_I64, _I64]),
    "qfp4_scales_bytes": (_SZ, [_I32, _I64, _I64]),
    "qfp4_scale_offset": (_I64, [_I32, _I64, _I64, _I64, _I64]),
    "qfp4_quantize_workspace_bytes": (_SZ, []),
    "qfp4_amax": (ctypes.c_int, [_VOID, _I64, _I64, _I64, _I32, _I32, ctypes.POINTER(Seed), _VOID, _VOID, _SZ, _VOID]),
    "qfp4_amax_rowcol": (ctypes.c_int, [_VOID, _I64, _I64, _I64, _I32, _I32, ctypes.POINTER(Seed), ctypes.POINTER(Seed),
                                        _VOID, _VOID, _VOID, _SZ, _VOID]),
    "qfp4_quantize": (ctypes.c_int, [_VOID, _I64, _I64, _I64, _I32, _I32, _I32, _I32, ctypes.POINTER(Seed), _VOID,
                                     ctypes.POINTER(TensorDesc), _VOID, _SZ, _VOID]),
    "qfp4_quantize_dual": (ctypes.c_int, [_VOID, _I64, _I64, _I64, _I32, _I32, _I32, _I32, ctypes.POINTER(Seed),
                                          ctypes.POINTER(Seed), _VOID, _VOID, ctypes.POINTER(TensorDesc),
                                          ctypes.POINTER(TensorDesc), _VOID]),
    "qfp4_gemm": (ctypes.c_int, [ctypes.POINTER(TensorDesc), ctypes.POINTER(TensorDesc), _VOID, _I64, _I32, _VOID]),
    "qfp4_gemm_quantize": (ctypes.c_int, [ctypes.POINTER(TensorDesc), ctypes.POINTER(TensorDesc), _VOID, _I64, _I32,
                                          ctypes.POINTER(Seed), ctypes.POINTER(TensorDesc), _VOID]),
    "qfp4_gemm_accumulate": (ctypes.c_int, [ctypes.POINTER(TensorDesc), ctypes.POINTER(TensorDesc), _VOID, _I64,
                                            _VOID]),
    "qfp4_gemm_amax": (ctypes.c_int, [ctypes.POINTER(TensorDesc), ctypes.POINTER(TensorDesc), _VOID, _I64, _I32,
                                      ctypes.POINTER(Seed), _VOID, _VOID, _SZ, _VOID]),
    "qfp4_recipe_preset": (ctypes.c_int, [_I32, ctypes.POINTER(Recipe)]),
    "qfp4_linear_workspace_bytes": (_SZ, [_I32, _I64, _I64, _I64, ctypes.POINTER(Recipe)]),
    "qfp4_linear_fwd": (ctypes.c_int, [_VOID, _VOID, _VOID, _I64, _I64, _I64, ctypes.POINTER(Recipe),
                                       ctypes.POINTER(Seed), _VOID, _SZ, _VOID]),
    "qfp4_linear_bwd": (ctypes.c_int, [_VOID, _VOID, _VOID, _VOID, _VOID, _I64, _I64, _I64, ctypes.POINTER(Recipe),
                                       ctypes.POINTER(Seed), _VOID, _SZ, _VOID]),
    "qfp4_linear_fwd_chain": (ctypes.c_int, [_VOID, _VOID, _VOID, _I64, _I64, _I64, ctypes.POINTER(Recipe),
                                             ctypes.POINTER(Seed), _VOID, _I32, ctypes.POINTER(Seed), _VOID, _VOID,
                                             _SZ, _VOID]),
    "qfp4_linear_fwd_noalloc": (ctypes.c_int, [_VOID, _VOID, _VOID, _I64, _I64, _I64, ctypes.POINTER(Recipe),
                                               ctypes.POINTER(Seed), _VOID]),
    "qfp4_status": (ctypes.c_int, [_VOID]),
    "qfp4_selftest_wait_timeout": (ctypes.c_int, [_I64, _VOID]),
    "qfp4_selftest_rounding": (ctypes.c_int, [_I32, _VOID, _VOID, _VOID, _I64, _VOID]),
    "qfp4_launch_count": (_I64, [_I32]),
}


def lib() -> ctypes.CDLL:
    """Load libqfp4.so (built by ``fp4_precision_b200.build``). Raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m fp4_precision_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != OK:
        raise QFP4Error(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def make_seed(rot: int = 0, sr: int = 0, rot_stream: int = 0, sr_stream: int = 0) -> Seed:
    return Seed(rot, sr, rot_stream, sr_stream)


# ---------------------------------------------------------------------------
# sizes / layout helpers (host only)

def codes_bytes(rows: int, k: int) -> int:
    return lib().qfp4_codes_bytes(rows, k)


def scales_bytes(fmt: int, rows: int, k: int) -> int:
    return lib().qfp4_scales_bytes(fmt, rows, k)


def scale_offset(fmt: int, rows: int, k: int, r: int, c: int) -> int:
    return lib().qfp4_scale_offset(fmt, rows, k, r, c)


def quantize_workspace_bytes() -> int:
    return lib().qfp4_quantize_workspace_bytes()


def launch_count(reset: bool = False) -> int:
    return lib().qfp4_launch_count(1 if reset else 0)


# ---------------------------------------------------------------------------
@dataclass
class QTensor:
    """A quantized operand in device memory (see qfp4_tensor in include/qfp4.h)."""
    codes: torch.Tensor         # uint8 [rows, k/2]
    scales: torch.Tensor        # uint8 [scales_bytes], MMA atom layout
    tensor_scale: torch.Tensor  # float32 [1]
    desc: TensorDesc

    @property
    def rows(self) -> int:
        return self.desc.rows

    @property
    def k(self) -> int:
        return self.desc.k

    @property
    def fmt(self) -> int:
        return self.desc.fmt


def empty_qtensor(fmt: int, rows: int, k: int, device) -> QTensor:
    codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((max(scales_bytes(fmt, rows, k), 16),), dtype=torch.uint8, device=device)
    ts = torch.empty((1,), dtype=torch.float32, device=device)
    desc = TensorDesc(codes.data_ptr(), scales.data_ptr(), ts.data_ptr(), 0, 0, 0, 0, 0, 0, 0)
    return QTensor(codes, scales, ts, desc)


def amax(x: torch.Tensor, had: int = HAD_NONE, axis: int = ROW, seed: Seed | None = None, out=None,
         workspace=None, stream=None) -> torch.Tensor:
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    R, C = x.shape
    out = torch.empty((1,), dtype=torch.float32, device=x.device) if out is None else out
    ws = torch.empty((quantize_workspace_bytes(),), dtype=torch.uint8, device=x.device) if workspace is None else workspace
    seed = seed or make_seed()
    _check(lib().qfp4_amax(_ptr(x), R, C, x.stride(0), had, axis, ctypes.byref(seed), _ptr(out), _ptr(ws),
                           ws.numel(), _stream(stream)), "qfp4_amax")
    return out


def amax_rowcol(x: torch.Tensor, had: int, seed_row: Seed | None = None, seed_col: Seed | None = None, out=None,
                workspace=None, stream=None, had_col: int | None = None) -> torch.Tensor:
    """Both orientations' tensor amax in one call: out[0] as amax(x, had, ROW,
    seed_row), out[1] as amax(x, had_col (default had), COL, seed_col)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    R, C = x.shape
    out = torch.empty((2,), dtype=torch.float32, device=x.device) if out is None else out
    ws = torch.empty((quantize_workspace_bytes(),), dtype=torch.uint8, device=x.device) if workspace is None else workspace
    seed_row = seed_row or make_seed()
    seed_col = seed_col or make_seed()
    had_col = had if had_col is None else had_col
    _check(lib().qfp4_amax_rowcol(_ptr(x), R, C, x.stride(0), had, had_col, ctypes.byref(seed_row),
                                  ctypes.byref(seed_col),
                                  _ptr(out), ctypes.c_void_p(out.data_ptr() + 4), _ptr(ws), ws.numel(),
                                  _stream(stream)), "qfp4_amax_rowcol")
    return out


def quantize(x: torch.Tensor, fmt: int, rounding: int, had: int, axis: int, seed: Seed | None = None,
             amax_in: torch.Tensor | None = None, out: QTensor | None = None, workspace=None,
             stream=None) -> QTensor:
    """Quantize a bf16 matrix (row stride x.stride(0)); see qfp4_quantize."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    R, C = x.shape
    rows, k = (R, C) if axis == ROW else (C, R)
    out = empty_qtensor(fmt, rows, k, x.device) if out is None else out
    ws = workspace
    if ws is None:
        ws = torch.empty((quantize_workspace_bytes(),), dtype=torch.uint8, device=x.device)
    seed = seed or make_seed()
    _check(lib().qfp4_quantize(_ptr(x), R, C, x.stride(0), fmt, rounding, had, axis, ctypes.byref(seed),
                               _ptr(amax_in), ctypes.byref(out.desc), _ptr(ws), ws.numel(), _stream(stream)),
           "qfp4_quantize")
    return out


def quantize_dual(x: torch.Tensor, fmt: int, rounding: int, had_row: int, had_col: int, seed_row: Seed,
                  seed_col: Seed, amax_row: torch.Tensor | None = None, amax_col: torch.Tensor | None = None,
                  out_row: QTensor | None = None, out_col: QTensor | None = None, stream=None):
    """Row and column quantization of a bf16 matrix from one read; see qfp4_quantize_dual."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    R, C = x.shape
    out_row = empty_qtensor(fmt, R, C, x.device) if out_row is None else out_row
    out_col = empty_qtensor(fmt, C, R, x.device) if out_col is None else out_col
    _check(lib().qfp4_quantize_dual(_ptr(x), R, C, x.stride(0), fmt, rounding, had_row, had_col,
                                    ctypes.byref(seed_row), ctypes.byref(seed_col), _ptr(amax_row), _ptr(amax_col),
                                    ctypes.byref(out_row.desc), ctypes.byref(out_col.desc), _stream(stream)),
           "qfp4_quantize_dual")
    return out_row, out_col


def gemm(A: QTensor, B: QTensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    """D = gA gB A . B^T (A.rows x B.rows); see qfp4_gemm."""
    dt = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    if out is None:
        out = torch.empty((A.rows, B.rows), dtype=out_dtype, device=A.codes.device)
    _check(lib().qfp4_gemm(ctypes.byref(A.desc), ctypes.byref(B.desc), _ptr(out), out.stride(0), dt,
                           _stream(stream)), "qfp4_gemm")
    return out


def gemm_quantize(A: QTensor, B: QTensor, had: int, seed: Seed, out: torch.Tensor | None = None,
                  qout: QTensor | None = None, stream=None):
    """bf16 D = gA gB A . B^T and its MXFP4 quantization along N; see qfp4_gemm_quantize."""
    if out is None:
        out = torch.empty((A.rows, B.rows), dtype=torch.bfloat16, device=A.codes.device)
    qout = empty_qtensor(MXFP4, A.rows, B.rows, A.codes.device) if qout is None else qout
    _check(lib().qfp4_gemm_quantize(ctypes.byref(A.desc), ctypes.byref(B.desc), _ptr(out), out.stride(0), had,
                                    ctypes.byref(seed), ctypes.byref(qout.desc), _stream(stream)),
           "qfp4_gemm_quantize")
    return out, qout


def gemm_amax(A: QTensor, B: QTensor, had: int, seed: Seed | None = None, out: torch.Tensor | None = None,
              amax: torch.Tensor | None = None, workspace=None, stream=None):
    """bf16 D = gA gB A . B^T and the NVFP4 tensor amax of D along its rows
    after the rotation `had`; see qfp4_gemm_amax. Returns (D, amax)."""
    if out is None:
        out = torch.empty((A.rows, B.rows), dtype=torch.bfloat16, device=A.codes.device)
    amax = torch.empty((1,), dtype=torch.float32, device=A.codes.device) if amax is None else amax
    ws = workspace
    if ws is None:
        ws = torch.empty((quantize_workspace_bytes(),), dtype=torch.uint8, device=A.codes.device)
    seed = seed or make_seed()
    _check(lib().qfp4_gemm_amax(ctypes.byref(A.desc), ctypes.byref(B.desc), _ptr(out), out.stride(0), had,
                                ctypes.byref(seed), _ptr(amax), _ptr(ws), ws.numel(), _stream(stream)),
           "qfp4_gemm_amax")
    return out, amax


def gemm_accumulate(A: QTensor, B: QTensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    """out += gA gB A . B^T in fp32 (A.rows x B.rows); see qfp4_gemm_accumulate."""
    assert out.dtype == torch.float32 and out.dim() == 2 and out.stride(1) == 1
    _check(lib().qfp4_gemm_accumulate(ctypes.byref(A.desc), ctypes.byref(B.desc), _ptr(out), out.stride(0),
                                      _stream(stream)), "qfp4_gemm_accumulate")
    return out


def recipe(name: str, dw_fp32: bool = True) -> Recipe:
    r = Recipe()
    _check(lib().qfp4_recipe_preset(PRESETS[name], ctypes.byref(r)), "qfp4_recipe_preset")
    r.dw_dtype = OUT_F32 if dw_fp32 else OUT_BF16
    return r


def linear_workspace_bytes(backward: bool, M: int, N: int, K: int, rec: Recipe) -> int:
    return lib().qfp4_linear_workspace_bytes(1 if backward else 0, M, N, K, ctypes.byref(rec))


def _dtype(code: int):
    return torch.float32 if code == OUT_F32 else torch.bfloat16


def linear_fwd(X, W, rec: Recipe, seed: Seed, Y=None, workspace=None, stream=None) -> torch.Tensor:
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty((M, N), dtype=_dtype(rec.y_dtype), device=X.device) if Y is None else Y
    if workspace is None:
        workspace = torch.empty((linear_workspace_bytes(False, M, N, K, rec),), dtype=torch.uint8, device=X.device)
    _check(lib().qfp4_linear_fwd(_ptr(X), _ptr(W), _ptr(Y), M, N, K, ctypes.byref(rec), ctypes.byref(seed),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "qfp4_linear_fwd")
    return Y


def linear_fwd_chain(X, W, rec: Recipe, seed: Seed, x_amax=None, next_had: int = HAD_NONE,
                     next_seed: Seed | None = None, want_y_amax: bool = True, Y=None, workspace=None, stream=None):
    """qfp4_linear_fwd_chain: the forward pass taking X's NVFP4 tensor amax
    (x_amax, from the previous layer) and returning Y's for the next layer's
    Fprop rotation (next_had, next_seed). Returns (Y, y_amax or None)."""
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty((M, N), dtype=_dtype(rec.y_dtype), device=X.device) if Y is None else Y
    if workspace is None:
        workspace = torch.empty((linear_workspace_bytes(False, M, N, K, rec),), dtype=torch.uint8, device=X.device)
    y_amax = torch.empty((1,), dtype=torch.float32, device=X.device) if want_y_amax else None
    ns = ctypes.byref(next_seed) if next_seed is not None else None
    _check(lib().qfp4_linear_fwd_chain(_ptr(X), _ptr(W), _ptr(Y), M, N, K, ctypes.byref(rec), ctypes.byref(seed),
                                       _ptr(x_amax), next_had, ns, _ptr(y_amax), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "qfp4_linear_fwd_chain")
    return Y, y_amax


def linear_fwd_noalloc(X, W, rec: Recipe, seed: Seed, Y=None, stream=None) -> torch.Tensor:
    """qfp4_linear_fwd_noalloc: the forward pass with the library's fixed
    scratch instead of a workspace (the binding allocates Y only if not given)."""
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty((M, N), dtype=_dtype(rec.y_dtype), device=X.device) if Y is None else Y
    _check(lib().qfp4_linear_fwd_noalloc(_ptr(X), _ptr(W), _ptr(Y), M, N, K, ctypes.byref(rec), ctypes.byref(seed),
                                         _stream(stream)), "qfp4_linear_fwd_noalloc")
    return Y


def linear_bwd(dY, X, W, rec: Recipe, seed: Seed, dX=None, dW=None, workspace=None, stream=None):
    M, K = X.shape
    N = W.shape[0]
    dX = torch.empty((M, K), dtype=_dtype(rec.dx_dtype), device=X.device) if dX is None else dX
    if rec.dw_accumulate and dW is None:
        raise ValueError("a recipe with dw_accumulate adds into dW: pass the buffer")
    dW = torch.empty((N, K), dtype=_dtype(rec.dw_dtype), device=X.device) if dW is None else dW
    if workspace is None:
        workspace = torch.empty((linear_workspace_bytes(True, M, N, K, rec),), dtype=torch.uint8, device=X.device)
    _check(lib().qfp4_linear_bwd(_ptr(dY), _ptr(X), _ptr(W), _ptr(dX), _ptr(dW), M, N, K, ctypes.byref(rec),
                                 ctypes.byref(seed), _ptr(workspace), workspace.numel(), _stream(stream)),
           "qfp4_linear_bwd")
    return dX, dW


def status(stream=None):
    """Synchronize and raise if a kernel reported a device-side error."""
    _check(lib().qfp4_status(_stream(stream)), "qfp4_status")


def selftest_rounding(op: int, x: torch.Tensor, w: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The quantizers' rounding step `op` (ROUND_*) applied to each fp32 of x
    with the uint32 random words w (int32 storage): one code byte per value."""
    assert x.dtype == torch.float32 and x.is_contiguous()
    assert w is None or (w.dtype == torch.int32 and w.is_contiguous() and w.numel() == x.numel())
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().qfp4_selftest_rounding(op, _ptr(x), _ptr(w), _ptr(codes), x.numel(), _stream(stream)),
           "qfp4_selftest_rounding")
    return codes


class Fp4Linear(torch.autograd.Function):
    """y = x W^T with FP4 Fprop/Dgrad/Wgrad (bf16 inputs, recipe + seed per call)."""

    @staticmethod
    def forward(ctx, X, W, rec: Recipe, seed: Seed):
        ctx.save_for_backward(X, W)
        ctx.rec, ctx.seed = rec, seed
        return linear_fwd(X.contiguous(), W.contiguous(), rec, seed)

    @staticmethod
    def backward(ctx, dY):
        X, W = ctx.saved_tensors
        dX, dW = linear_bwd(dY.contiguous().to(torch.bfloat16), X.contiguous(), W.contiguous(), ctx.rec, ctx.seed)
        return dX.to(X.dtype), dW.to(W.dtype), None, None
