"""Quantization past 32-bit indices: a [139264 x 32768] bf16 tensor (4.56e9
elements, 9.1 GB). One quantization's codes span 2.28 GB, so byte offsets
pass 2^31, and the element indices that address the stochastic-rounding
words pass 2^32 (row-major index r * k + c of the quantized orientation).
NVFP4 with per-element SR and with Quartet II, no rotation, along rows and
along columns; sampled rows of the quantized orientation (first and last,
around element 2^31 and 2^32, random) match the oracle bit for bit, codes,
scales and tensor scale. The oracle takes the tensor amax max |x| (the
definition without a rotation) from the host copy and quantizes only the
sampled rows, with the random words of their own indices."""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

import helpers

pytestmark = pytest.mark.gpu

R, C = 139264, 32768
ROT, SR = 0x0123_4567, 0x89AB_CDEF


def sampled(n, k, rng):
    """Rows of a [n x k] orientation: the ends, the rows whose element index
    crosses 2^31 and 2^32, and random ones."""
    cross = [(1 << 31) // k, (1 << 32) // k]
    fixed = [0, 1, n - 2, n - 1] + [r + d for r in cross for d in (-1, 0, 1)]
    rest = rng.choice(n, size=8, replace=False)
    return np.unique(np.clip(np.concatenate([fixed, rest]), 0, n - 1))


def assert_rows_same(q_gpu, q_ref, rows):
    codes = q_gpu.codes.index_select(0, torch.as_tensor(rows, device=q_gpu.codes.device)).cpu().numpy()
    assert np.array_equal(codes, q_ref.codes), f"{np.sum(codes != q_ref.codes)} code bytes differ"
    flat = helpers.to_numpy_u8(q_gpu.scales)
    kb = q_gpu.k // 16
    sc = flat[helpers.atom_offset(q_gpu.rows, kb, np.asarray(rows, dtype=np.int64)[:, None],
                                  np.arange(kb, dtype=np.int64)[None, :])]
    assert np.array_equal(sc, q_ref.scales), f"{np.sum(sc != q_ref.scales)} scales differ"
    g = float(q_gpu.tensor_scale.cpu()[0])
    assert np.float32(g).tobytes() == np.float32(q_ref.g).tobytes(), (g, q_ref.g)


def test_quantize_past_32_bit_indices():
    free, _ = torch.cuda.mem_get_info()
    if free < 40 * 2**30:
        pytest.skip("needs about 40 GB of free device memory")
    dev = torch.device("cuda", 0)
    x = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
    for i in range(0, R, 8192):  # drawn in slices: no 18 GB fp32 temporary
        x[i:i + 8192] = inputs.normal((8192, C), 1.0, 31 + i // 8192, "large", device=dev)
    x_cpu = x.cpu()
    amax = max(float(x_cpu[i:i + 8192].abs().max()) for i in range(0, R, 8192))
    rng = np.random.default_rng(3)
    for rnd in (Q.SR, Q.QUARTET2):
        for axis in (Q.ROW, Q.COL):
            seed = Q.make_seed(ROT, SR, 1, 5 + axis)
            q = Q.quantize(x, Q.NVFP4, rnd, Q.HAD_NONE, axis, seed)
            torch.cuda.synchronize()
            Q.status()
            rows = sampled(q.rows, q.k, rng)
            ref = O.quantize(x_cpu, Q.NVFP4, rnd, Q.HAD_NONE, axis, ROT, 1, SR, 5 + axis, amax=amax, rows_sel=rows)
            assert_rows_same(q, ref, rows)
            del q


def test_gemm_past_31_bit_output_offsets():
    """GEMM outputs past 2^31 bytes: D [40960 x 28672] in bf16 (2.35 GB) and in
    fp32 (4.70 GB) from NVFP4 operands with K = 256, and the fp32 output again
    accumulated into (D += A B^T). Sampled outputs around the row where the
    byte offset crosses 2^31, and at the ends, are within 2^-18 * sum |a b| of
    fp64 dot products of the oracle's quantization of the sampled rows (bf16
    outputs add 2^-8 |D|)."""
    M, N, K = 40960, 28672, 256
    free, _ = torch.cuda.mem_get_info()
    if free < 24 * 2**30:
        pytest.skip("needs about 24 GB of free device memory")
    dev = torch.device("cuda", 0)
    A = inputs.normal((M, K), 1.0, 41, "A", device=dev)
    B = inputs.normal((N, K), 1.0, 41, "B", device=dev)
    seed_a, seed_b = Q.make_seed(ROT, SR, 0, 0), Q.make_seed(ROT, SR, 0, 1)
    qa = Q.quantize(A, Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW, seed_a)
    qb = Q.quantize(B, Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW, seed_b)
    rng = np.random.default_rng(5)
    ra = np.unique(np.concatenate([[0, 1, M - 1], [r + d for r in ((1 << 29) // N, (1 << 30) // N) for d in (-1, 0, 1)],
                                   rng.choice(M, 8, replace=False)]))
    rb = np.unique(np.concatenate([[0, 1, N // 2, N - 1], rng.choice(N, 12, replace=False)]))
    Ad = O.dequantize(O.quantize(A.cpu(), Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW, ROT, 0, SR, 0, rows_sel=ra))
    Bd = O.dequantize(O.quantize(B.cpu(), Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW, ROT, 0, SR, 1, rows_sel=rb))
    ref = Ad @ Bd.T
    bound = O.GEMM_REL_BOUND * (np.abs(Ad) @ np.abs(Bd).T)
    ia, ib = torch.as_tensor(ra, device=dev), torch.as_tensor(rb, device=dev)

    def check(D, tol, what):
        got = D.index_select(0, ia).index_select(1, ib).double().cpu().numpy()
        err = np.abs(got - ref)
        assert np.all(err <= tol), f"{what}: {np.sum(err > tol)} of {err.size} sampled outputs out of bound"

    D = Q.gemm(qa, qb, torch.bfloat16)
    torch.cuda.synchronize()
    Q.status()
    check(D, bound + 2.0 ** -8 * np.abs(ref), "bf16")
    del D
    D = Q.gemm(qa, qb, torch.float32)
    torch.cuda.synchronize()
    Q.status()
    check(D, bound, "fp32")
    Q.gemm_accumulate(qa, qb, D)
    torch.cuda.synchronize()
    Q.status()
    ref = 2.0 * ref
    check(D, 2.0 * bound + np.abs(ref) * 2.0 ** -24, "fp32 accumulated")
