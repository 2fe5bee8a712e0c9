"""GPU block-scaled FP4 GEMMs vs the fp64 oracle, within
|err| <= 2^-18 * sum_k |a_k b_k| per element (fp32 output; a bf16 output adds
its own rounding, 2^-8 |D|). The GEMM is fed the oracle's own quantized
operands (codes, scales and tensor scales laid out as include/qfp4.h states),
so these tests isolate the GEMM from the quantizers."""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

import helpers

pytestmark = pytest.mark.gpu


def upload(qo: O.QTensor, rot_seed=0, rot_stream=0) -> Q.QTensor:
    """An oracle-quantized operand as a device QTensor."""
    nb = O.BLOCK[qo.fmt]
    kb = qo.k // nb
    nbytes = max(Q.scales_bytes(qo.fmt, qo.rows, qo.k), 16)
    flat = np.zeros(nbytes, dtype=np.uint8)
    r = np.arange(qo.rows)[:, None]
    c = np.arange(kb)[None, :]
    flat[helpers.atom_offset(qo.rows, kb, r, c)] = qo.scales
    codes = torch.from_numpy(qo.codes.copy()).cuda()
    scales = torch.from_numpy(flat).cuda()
    ts = torch.tensor([qo.g], dtype=torch.float32, device="cuda")
    desc = Q.TensorDesc(codes.data_ptr(), scales.data_ptr(), ts.data_ptr(), qo.rows, qo.k, qo.fmt, qo.had,
                        rot_seed, rot_stream, 0)
    return Q.QTensor(codes, scales, ts, desc)


def check_gemm(A_o, B_o, out_dtype, rows=None, cols=None, rot=(0, 0)):
    A, B = upload(A_o, *rot), upload(B_o, *rot)
    D, guard = helpers.guarded_matrix(A.rows, B.rows, out_dtype, "cuda")
    Q.gemm(A, B, out_dtype, out=D)
    torch.cuda.synchronize()
    Q.status()
    helpers.assert_guards_intact(guard)
    Dg = D.float().cpu().numpy().astype(np.float64)
    if rows is None:
        ref, bound = O.gemm(A_o, B_o), O.gemm_bound(A_o, B_o)
    else:
        Ad, Bd = O.dequantize(A_o)[rows], O.dequantize(B_o)[cols]
        ref = np.einsum("ik,ik->i", Ad, Bd)
        bound = O.GEMM_REL_BOUND * np.einsum("ik,ik->i", np.abs(Ad), np.abs(Bd))
        Dg = Dg[rows, cols]
    tol = bound + (2.0 ** -8 * np.abs(ref) if out_dtype == torch.bfloat16 else 0.0)
    err = np.abs(Dg - ref)
    worst = np.max(err / np.maximum(bound / O.GEMM_REL_BOUND, 1e-300))
    assert np.all(err <= tol), f"{np.sum(err > tol)} outputs out of bound; max err/sum|ab| = {worst:.3e}"
    return worst


@pytest.fixture(params=["pair", "single", "default"])
def kernel_variant(request, monkeypatch):
    """Both GEMM kernels, forced (the CTA pair, the single CTA), and the
    library's own choice (the pair when A has more than 128 rows)."""
    if request.param == "pair":
        monkeypatch.setenv("QFP4_GEMM_PAIR", "1")
    elif request.param == "single":
        monkeypatch.setenv("QFP4_GEMM_PAIR", "0")
    else:
        monkeypatch.delenv("QFP4_GEMM_PAIR", raising=False)
    return request.param


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4], ids=["nvfp4", "mxfp4"])
@pytest.mark.parametrize("shape", [(128, 256, 256), (300, 200, 320), (512, 520, 1024), (100, 136, 192)],
                         ids=lambda s: "x".join(map(str, s)))
def test_gemm_accumulate_matches_oracle(fmt, shape, kernel_variant):
    """D += A . B^T into an fp32 buffer (beta = 1): the product within the
    GEMM bound, then one fp32 add per element; untouched outside A.rows x
    B.rows (a wider row stride leaves the padding columns as they were)."""
    M, N, K = shape
    X = inputs.normal_with_outliers((M, K), 23, "aa")
    W = inputs.normal((N, K), 0.02, 23, "ab")
    A_o = O.quantize(X, fmt, O.RTN, O.HAD_NONE, O.ROW)
    B_o = O.quantize(W, fmt, O.SR, O.HAD_NONE, O.ROW, 0, 0, 5, 1)
    A, B = upload(A_o), upload(B_o)
    ld = N + 4 - N % 4 + 8
    D0 = inputs.normal((M, ld), 3.0, 23, "d0").float().cuda()
    D = D0.clone()
    Q.gemm_accumulate(A, B, D[:, :N])
    torch.cuda.synchronize()
    Q.status()
    ref = O.gemm(A_o, B_o)
    d0 = D0[:, :N].cpu().numpy().astype(np.float64)
    tol = O.gemm_bound(A_o, B_o) + 2.0 ** -23 * (np.abs(d0) + np.abs(ref))
    err = np.abs(D[:, :N].cpu().numpy().astype(np.float64) - (d0 + ref))
    assert np.all(err <= tol), f"{np.sum(err > tol)} outputs out of bound"
    assert torch.equal(D[:, N:], D0[:, N:])
    # twice: the second call adds the same product again
    Q.gemm_accumulate(A, B, D[:, :N])
    torch.cuda.synchronize()
    err2 = np.abs(D[:, :N].cpu().numpy().astype(np.float64) - (d0 + 2 * ref))
    assert np.all(err2 <= 2 * tol + 2.0 ** -23 * np.abs(d0 + 2 * ref))


def grid_operand(rows, k, seed):
    """bf16 [rows, k] of E2M1 grid values with a +-6 in every 32-element block
    along k: its MXFP4 RTN quantization is exact with every scale 2^0."""
    g = np.random.default_rng(seed)
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    x = vals[g.integers(0, 8, size=(rows, k))] * np.where(g.random((rows, k)) < 0.5, -1.0, 1.0)
    x[:, ::32] = 6.0 * np.where(g.random((rows, k // 32)) < 0.5, -1.0, 1.0)
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("had", [O.HAD_NONE, O.HAD_DET16, O.HAD_DET32, O.HAD_RAND16, O.HAD_RAND32],
                         ids=["none", "det16", "det32", "rand16", "rand32"])
@pytest.mark.parametrize("shape", [(300, 288, 256), (128, 256, 128), (512, 1024, 512)],
                         ids=lambda s: "x".join(map(str, s)))
def test_gemm_quantize_matches_oracle(shape, had, kernel_variant):
    """qfp4_gemm_quantize: the bf16 output and its MXFP4 quantization along N.
    The operands are exactly representable and every partial sum is exact in
    fp32, so D is known exactly: the bf16 D must equal bf16(D) and the
    quantized output the oracle's quantization of it, bit for bit (rows and
    scale columns past the tensor included as zero padding)."""
    M, N, K = shape
    X, W = grid_operand(M, K, 1), grid_operand(N, K, 2)
    A_o = O.quantize(X, O.MXFP4, O.RTN, O.HAD_NONE, O.ROW)
    B_o = O.quantize(W, O.MXFP4, O.RTN, O.HAD_NONE, O.ROW)
    assert np.all(A_o.scales == 127) and np.all(B_o.scales == 127)
    d_exact = X.double().numpy() @ W.double().numpy().T
    d_bf16 = torch.from_numpy(d_exact.astype(np.float32)).to(torch.bfloat16)
    ref = O.quantize(d_bf16, O.MXFP4, O.RTN, had, O.ROW, 0x77, 5)
    Dg, g_d = helpers.guarded_matrix(M, N, torch.bfloat16, "cuda")
    qg, g_q = helpers.guarded_qtensor(Q, Q.MXFP4, M, N, "cuda")
    D, q = Q.gemm_quantize(upload(A_o), upload(B_o), had, Q.make_seed(rot=0x77, rot_stream=5), out=Dg, qout=qg)
    torch.cuda.synchronize()
    Q.status()
    helpers.assert_guards_intact(g_d, g_q)
    assert torch.equal(D.cpu(), d_bf16)
    assert q.fmt == Q.MXFP4 and q.rows == M and q.k == N
    codes = helpers.to_numpy_u8(q.codes)
    assert np.array_equal(codes, ref.codes), f"{np.sum(codes != ref.codes)} code bytes differ"
    flat = helpers.to_numpy_u8(q.scales)
    assert np.array_equal(helpers.unswizzle_scales(flat, M, N, 32), ref.scales)
    assert helpers.padding_is_zero(flat, M, N, 32)
    assert float(q.tensor_scale.cpu()[0]) == 1.0


@pytest.mark.parametrize("had", [O.HAD_NONE, O.HAD_RAND32], ids=["none", "rand32"])
def test_gemm_quantize_equals_quantizing_the_output(had):
    """With NVFP4 operands and a general K the fused quantization equals the
    row quantizer run on the GEMM's own bf16 output (same stream of values)."""
    M, N, K = 640, 544, 1024
    X = inputs.normal_with_outliers((M, K), 31, "qa")
    W = inputs.normal((N, K), 0.02, 31, "qb")
    A = upload(O.quantize(X, O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    B = upload(O.quantize(W, O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    seed = Q.make_seed(rot=0x55, rot_stream=2)
    D, q = Q.gemm_quantize(A, B, had, seed)
    q2 = Q.quantize(D, Q.MXFP4, Q.RTN, had, Q.ROW, seed)
    torch.cuda.synchronize()
    Q.status()
    assert torch.equal(q.codes, q2.codes) and torch.equal(q.scales, q2.scales)


def test_linear_dw_accumulate_needs_fp32_dw():
    """A recipe that accumulates into dW must have an fp32 dW: the call is
    rejected on the host, before anything is launched."""
    rec = Q.recipe("QUARTET2_NVFP4", dw_fp32=False)
    rec.dw_accumulate = 1
    X = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    dW = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Q.QFP4Error):
        Q.linear_bwd(X, X, X, rec, Q.make_seed(), dW=dW)
    acc = Q.recipe("QUARTET2_NVFP4")
    acc.dw_accumulate = 1
    with pytest.raises(ValueError):  # nothing to add into
        Q.linear_bwd(X, X, X, acc, Q.make_seed())


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4], ids=["nvfp4", "mxfp4"])
@pytest.mark.parametrize("shape", [(128, 256, 256), (300, 200, 320), (512, 520, 1024), (130, 640, 64),
                                   (1024, 768, 2048), (100, 136, 192)], ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_gemm_matches_oracle(fmt, shape, out_dtype, kernel_variant):
    M, N, K = shape
    X = inputs.normal_with_outliers((M, K), 21, "ga")
    W = inputs.normal((N, K), 0.02, 21, "gb")
    A_o = O.quantize(X, fmt, O.RTN, O.HAD_NONE, O.ROW)
    B_o = O.quantize(W, fmt, O.SR, O.HAD_NONE, O.ROW, 0, 0, 5, 1)
    check_gemm(A_o, B_o, out_dtype)


def test_gemm_rotated_operands(kernel_variant):
    """Random-Hadamard operands (same sign vector): the GEMM estimates X W^T."""
    M, N, K = 256, 512, 512
    X = inputs.normal((M, K), 1.0, 22, "ra")
    W = inputs.normal((N, K), 1.0, 22, "rb")
    A_o = O.quantize(X, O.NVFP4, O.QUARTET2, O.HAD_RAND16, O.ROW, 9, 1, 3, 0)
    B_o = O.quantize(W, O.NVFP4, O.QUARTET2, O.HAD_RAND16, O.ROW, 9, 1, 3, 1)
    check_gemm(A_o, B_o, torch.float32, rot=(9, 1))


def test_gemm_qkv_shape_sampled(kernel_variant):
    """The QKV-projection Fprop shape, 8192 x 6144 x 4096, in the launch
    configuration the benchmark times: 4096 sampled outputs plus two full
    128 x 128 tiles against fp64 dot products."""
    M, N, K = 8192, 6144, 4096
    wl = inputs.workload("qkv")
    A_o = O.quantize(wl["X"], O.NVFP4, O.RTN, O.HAD_DET16, O.ROW)
    B_o = O.quantize(wl["W"], O.NVFP4, O.RTN, O.HAD_DET16, O.ROW)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, M, 4096)
    cols = rng.integers(0, N, 4096)
    t = np.arange(128)
    rows = np.concatenate([rows, np.repeat(t, 128), np.repeat(8064 + t, 128)])
    cols = np.concatenate([cols, np.tile(t, 128), np.tile(6016 + t, 128)])
    worst = check_gemm(A_o, B_o, torch.float32, rows=rows, cols=cols)
    print(f"max err / sum|ab| = {worst:.3e}")


def test_gemm_rejects_mismatched_operands():
    X = inputs.normal((128, 256), 1.0, 23, "ma")
    A = upload(O.quantize(X, O.NVFP4, O.RTN, O.HAD_RAND16, O.ROW, 1, 0), 1, 0)
    B = upload(O.quantize(X, O.NVFP4, O.RTN, O.HAD_RAND16, O.ROW, 2, 0), 2, 0)
    with pytest.raises(Q.QFP4Error) as e:
        Q.gemm(A, B)
    assert e.value.status == Q.ERR_INVALID_ARG
    C = upload(O.quantize(X, O.MXFP4, O.RTN, O.HAD_RAND16, O.ROW, 1, 0), 1, 0)
    with pytest.raises(Q.QFP4Error):
        Q.gemm(A, C)


@pytest.mark.parametrize("had", [O.HAD_NONE, O.HAD_DET16, O.HAD_RAND16, O.HAD_RAND32],
                         ids=["none", "det16", "rand16", "rand32"])
@pytest.mark.parametrize("shape", [(300, 288, 256), (128, 256, 128), (640, 544, 1024), (1024, 2080, 512)],
                         ids=lambda s: "x".join(map(str, s)))
def test_gemm_amax_matches_oracle(shape, had, kernel_variant):
    """qfp4_gemm_amax: the bf16 D is exactly qfp4_gemm's, and the amax is the
    NVFP4 tensor amax of that D along its rows after the rotation (the
    oracle's max |rotated D|, bit for bit); quantizing D with it gives the
    same operand as quantizing D with its own amax pass. Ragged tiles in both
    directions, outputs between guard bytes."""
    M, N, K = shape
    X = inputs.normal_with_outliers((M, K), 41, "ga")
    W = inputs.normal((N, K), 0.02, 41, "gb")
    A = upload(O.quantize(X, O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    B = upload(O.quantize(W, O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    seed = Q.make_seed(rot=0x99, rot_stream=4)
    Dg, g_d = helpers.guarded_matrix(M, N, torch.bfloat16, "cuda")
    am = torch.full((1,), -1.0, device="cuda")
    D, am = Q.gemm_amax(A, B, had, seed, out=Dg, amax=am)
    D_ref = Q.gemm(A, B, torch.bfloat16)
    torch.cuda.synchronize()
    Q.status()
    helpers.assert_guards_intact(g_d)
    assert torch.equal(D, D_ref)
    v = O.rotate(D.cpu(), had, O.ROW, 0x99, 4)
    assert np.float32(am.cpu()[0]).tobytes() == np.float32(np.abs(v).max()).tobytes()
    assert float(Q.amax(D, had, Q.ROW, seed).cpu()[0]) == float(am.cpu()[0])
    q1 = Q.quantize(D, Q.NVFP4, Q.RTN, had, Q.ROW, seed, amax_in=am)
    q2 = Q.quantize(D, Q.NVFP4, Q.RTN, had, Q.ROW, seed)
    torch.cuda.synchronize()
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.scales, q2.scales)
    assert torch.equal(q1.tensor_scale, q2.tensor_scale)


def test_gemm_amax_rejects_bad_arguments():
    A = upload(O.quantize(inputs.normal((256, 128), 1.0, 3, "ra"), O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    B = upload(O.quantize(inputs.normal((200, 128), 1.0, 3, "rb"), O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    with pytest.raises(Q.QFP4Error):  # B.rows (the next layer's k) not a multiple of 16
        Q.gemm_amax(A, B, Q.HAD_NONE)
    B2 = upload(O.quantize(inputs.normal((208, 128), 1.0, 3, "rb"), O.NVFP4, O.RTN, O.HAD_NONE, O.ROW))
    with pytest.raises(Q.QFP4Error):  # ... nor of the Hadamard size
        Q.gemm_amax(A, B2, Q.HAD_RAND32, Q.make_seed(1))
    torch.cuda.synchronize()
