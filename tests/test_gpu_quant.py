"""GPU quantizers vs the CPU oracle: codes, scales and the tensor scale must
match bit for bit, for every format, rounding mode, Hadamard setting and
orientation, on ragged shapes, at the sweep workload's full size, and on the
degenerate inputs of the method."""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

import helpers

pytestmark = pytest.mark.gpu

HADS = [Q.HAD_NONE, Q.HAD_DET16, Q.HAD_DET32, Q.HAD_RAND16, Q.HAD_RAND32]
SEED = dict(rot=0x5EED_0001_2345_6789, sr=0xABCD_EF01_2345_6789, rot_stream=3, sr_stream=7)


def gpu_quant(x_dev, fmt, rnd, had, axis, **kw):
    """Quantize on the GPU into guarded output buffers and check that no byte
    outside codes, scales and tensor scale changed."""
    seed = Q.make_seed(**SEED)
    R, C = x_dev.shape
    rows, k = (R, C) if axis == Q.ROW else (C, R)
    out, guards = helpers.guarded_qtensor(Q, fmt, rows, k, x_dev.device)
    q = Q.quantize(x_dev, fmt, rnd, had, axis, seed, out=out, **kw)
    torch.cuda.synchronize()
    Q.status()
    helpers.assert_guards_intact(guards)
    return q


def oracle_quant(x_cpu, fmt, rnd, had, axis, amax=None):
    return O.quantize(x_cpu, fmt, rnd, had, axis, SEED["rot"], SEED["rot_stream"], SEED["sr"], SEED["sr_stream"],
                      amax=amax)


def assert_same(q_gpu, q_ref, fmt):
    nb = Q.BLOCK[fmt]
    codes = helpers.to_numpy_u8(q_gpu.codes)
    assert codes.shape == q_ref.codes.shape
    bad = np.argwhere(codes != q_ref.codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    flat = helpers.to_numpy_u8(q_gpu.scales)
    sc = helpers.unswizzle_scales(flat, q_ref.rows, q_ref.k, nb)
    bad = np.argwhere(sc != q_ref.scales)
    assert bad.size == 0, f"{len(bad)} scales differ, first at {bad[:5].tolist()}"
    assert helpers.padding_is_zero(flat, q_ref.rows, q_ref.k, nb)
    g = float(q_gpu.tensor_scale.cpu()[0])
    assert np.float32(g).tobytes() == np.float32(q_ref.g).tobytes(), (g, q_ref.g)


def sweep_like(R, C, seed=1):
    x = inputs.student_t_colgain((R, C), seed, "T")
    # a few large outliers so some blocks saturate and the tensor amax is far from typical
    x.view(-1)[:: 997] *= 40
    return x


@pytest.mark.parametrize("axis", [Q.ROW, Q.COL], ids=["row", "col"])
@pytest.mark.parametrize("had", HADS, ids=["none", "det16", "det32", "rand16", "rand32"])
@pytest.mark.parametrize("rnd", [Q.RTN, Q.SR, Q.QUARTET2], ids=["rtn", "sr", "q2"])
@pytest.mark.parametrize("fmt", [Q.NVFP4, Q.MXFP4, Q.MXFP4_RU], ids=["nvfp4", "mxfp4", "mxfp4ru"])
def test_quantize_matches_oracle_ragged(fmt, rnd, had, axis):
    # 352 x 416: several 128-tiles plus ragged tails in both directions
    x = sweep_like(352, 416)
    q = gpu_quant(x.cuda(), fmt, rnd, had, axis)
    assert_same(q, oracle_quant(x, fmt, rnd, had, axis), fmt)


@pytest.mark.parametrize("shape", [(320, 424), (448, 136)], ids=["320x424", "448x136"])
@pytest.mark.parametrize("had", HADS, ids=["none", "det16", "det32", "rand16", "rand32"])
@pytest.mark.parametrize("rnd", [Q.RTN, Q.SR, Q.QUARTET2], ids=["rtn", "sr", "q2"])
@pytest.mark.parametrize("fmt", [Q.NVFP4, Q.MXFP4, Q.MXFP4_RU], ids=["nvfp4", "mxfp4", "mxfp4ru"])
def test_column_bands_match_oracle(fmt, rnd, had, shape, monkeypatch):
    """The column quantizer over 64-row bands (quantized axis a multiple of
    64): a partial last tile of 256 rows (320 = 5 bands; 448 = 7 bands, which
    also leaves half of the last MXFP4 scale word as padding) and a partial
    last tile of 64 columns; and the group-walking kernel on the same input."""
    x = sweep_like(*shape)
    ref = oracle_quant(x, fmt, rnd, had, Q.COL)
    assert_same(gpu_quant(x.cuda(), fmt, rnd, had, Q.COL), ref, fmt)
    monkeypatch.setenv("QFP4_COL_BANDS", "0")
    assert_same(gpu_quant(x.cuda(), fmt, rnd, had, Q.COL), ref, fmt)


DUAL_HADS = [(Q.HAD_NONE, Q.HAD_NONE), (Q.HAD_NONE, Q.HAD_RAND16), (Q.HAD_RAND16, Q.HAD_RAND16),
             (Q.HAD_DET16, Q.HAD_RAND16), (Q.HAD_NONE, Q.HAD_DET32), (Q.HAD_RAND32, Q.HAD_RAND32)]


@pytest.mark.parametrize("shape", [(320, 416), (448, 160)], ids=["320x416", "448x160"])
@pytest.mark.parametrize("hads", DUAL_HADS, ids=lambda h: f"row{h[0]}-col{h[1]}")
@pytest.mark.parametrize("rnd", [Q.RTN, Q.SR, Q.QUARTET2], ids=["rtn", "sr", "q2"])
@pytest.mark.parametrize("fmt", [Q.NVFP4, Q.MXFP4, Q.MXFP4_RU], ids=["nvfp4", "mxfp4", "mxfp4ru"])
def test_quantize_dual_matches_oracle(fmt, rnd, hads, shape):
    """Both orientations from one read (qfp4_quantize_dual) equal the oracle's
    row and column quantizations: partial last tiles in rows (5 or 7 bands of
    64) and columns, MXFP4 scale words half padding, different sign vectors
    and Hadamard sizes for the two orientations."""
    had_row, had_col = hads
    x = sweep_like(*shape)
    xd = x.cuda()
    s_row = Q.make_seed(SEED["rot"], SEED["sr"], 1, 2)
    s_col = Q.make_seed(SEED["rot"], SEED["sr"], 2, 4)
    am_row = am_col = None
    if fmt == Q.NVFP4:
        am_row = Q.amax(xd, had_row, Q.ROW, s_row)
        am_col = Q.amax(xd, had_col, Q.COL, s_col)
    R, C = shape
    out_row, g_row = helpers.guarded_qtensor(Q, fmt, R, C, xd.device)
    out_col, g_col = helpers.guarded_qtensor(Q, fmt, C, R, xd.device)
    qr, qc = Q.quantize_dual(xd, fmt, rnd, had_row, had_col, s_row, s_col, am_row, am_col, out_row=out_row,
                             out_col=out_col)
    torch.cuda.synchronize()
    Q.status()
    helpers.assert_guards_intact(g_row, g_col)
    assert qr.fmt == qc.fmt == (Q.MXFP4 if fmt == Q.MXFP4_RU else fmt)
    assert_same(qr, O.quantize(x, fmt, rnd, had_row, Q.ROW, SEED["rot"], 1, SEED["sr"], 2), fmt)
    assert_same(qc, O.quantize(x, fmt, rnd, had_col, Q.COL, SEED["rot"], 2, SEED["sr"], 4), fmt)


def test_quantize_dual_rejects_unsupported():
    x = sweep_like(128, 128).cuda()
    s = Q.make_seed(1, 2)
    with pytest.raises(Q.QFP4Error):  # rows not a multiple of 64
        Q.quantize_dual(x[:96], Q.MXFP4, Q.RTN, Q.HAD_NONE, Q.HAD_NONE, s, s)
    with pytest.raises(Q.QFP4Error):  # row Hadamard neither none nor the column one's size
        Q.quantize_dual(x, Q.MXFP4, Q.RTN, Q.HAD_DET16, Q.HAD_DET32, s, s)
    with pytest.raises(Q.QFP4Error):  # NVFP4 needs both tensor amaxes
        Q.quantize_dual(x, Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.HAD_NONE, s, s)
    torch.cuda.synchronize()


@pytest.mark.parametrize("axis", [Q.ROW, Q.COL], ids=["row", "col"])
@pytest.mark.parametrize("rnd", [Q.RTN, Q.SR, Q.QUARTET2], ids=["rtn", "sr", "q2"])
def test_nvfp4_axis_not_a_multiple_of_32(rnd, axis):
    """NVFP4 needs only k % 16 == 0: with k = 208 the codes of a row start
    8-byte aligned (the 32-byte code stores split into 8-byte ones)."""
    x = sweep_like(208, 208)
    for had in (Q.HAD_NONE, Q.HAD_DET16, Q.HAD_RAND16):
        q = gpu_quant(x.cuda(), Q.NVFP4, rnd, had, axis)
        assert_same(q, oracle_quant(x, Q.NVFP4, rnd, had, axis), Q.NVFP4)


@pytest.mark.parametrize("case", [
    (Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW), (Q.NVFP4, Q.QUARTET2, Q.HAD_RAND16, Q.COL),
    (Q.MXFP4, Q.SR, Q.HAD_DET32, Q.COL), (Q.NVFP4, Q.SR, Q.HAD_NONE, Q.ROW),
    (Q.MXFP4, Q.QUARTET2, Q.HAD_RAND32, Q.ROW), (Q.NVFP4, Q.RTN, Q.HAD_DET16, Q.COL),
    (Q.MXFP4_RU, Q.RTN, Q.HAD_DET32, Q.COL), (Q.MXFP4_RU, Q.SR, Q.HAD_NONE, Q.ROW),
    # Quartet II with no Hadamard: about one block in a million has its scale's
    # stochastic rounding within an ulp of alpha, so a product fused into the
    # alpha sums shows here (two blocks per orientation)
    (Q.NVFP4, Q.QUARTET2, Q.HAD_NONE, Q.ROW), (Q.NVFP4, Q.QUARTET2, Q.HAD_NONE, Q.COL),
    (Q.NVFP4, Q.QUARTET2, Q.HAD_RAND16, Q.ROW), (Q.MXFP4, Q.QUARTET2, Q.HAD_NONE, Q.COL),
], ids=lambda c: f"{['nv', 'mx', 'mxru'][c[0]]}-{['rtn', 'sr', 'q2'][c[1]]}-h{c[2]}-{['row', 'col'][c[3]]}")
def test_quantize_full_sweep_workload(case):
    """The quantizer-sweep workload at its full size, [8192 x 4096]."""
    fmt, rnd, had, axis = case
    x_dev = inputs.workload("sweep", device="cuda")["T"]
    q = gpu_quant(x_dev, fmt, rnd, had, axis)
    assert_same(q, oracle_quant(x_dev.cpu(), fmt, rnd, had, axis), fmt)


@pytest.mark.parametrize("fmt", [Q.NVFP4, Q.MXFP4])
@pytest.mark.parametrize("shape", [(32, 32), (1, 64), (33, 96), (128, 128), (16, 4096), (4096, 32)])
@pytest.mark.parametrize("axis", [Q.ROW, Q.COL])
def test_small_and_thin_shapes(fmt, shape, axis):
    R, C = shape
    x = inputs.normal_with_outliers((R, C), 5, "thin")
    rows_k = (R, C) if axis == Q.ROW else (C, R)
    if rows_k[1] % 32:
        pytest.skip("quantized axis must be a multiple of 32 for every Hadamard size")
    for rnd, had in ((Q.RTN, Q.HAD_NONE), (Q.QUARTET2, Q.HAD_RAND32), (Q.SR, Q.HAD_DET16)):
        q = gpu_quant(x.cuda(), fmt, rnd, had, axis)
        assert_same(q, oracle_quant(x, fmt, rnd, had, axis), fmt)


def test_mxfp4_round_up_writes_an_mxfp4_tensor():
    """The round-up variant only changes the shared exponent: the tensor it
    writes is an ordinary MXFP4 tensor (format field, scale layout), its
    exponents are the floor rule's or one more, and a GEMM takes it."""
    x_dev = sweep_like(256, 512).cuda()
    qf = gpu_quant(x_dev, Q.MXFP4, Q.RTN, Q.HAD_NONE, Q.ROW)
    qr = gpu_quant(x_dev, Q.MXFP4_RU, Q.RTN, Q.HAD_NONE, Q.ROW)
    assert qr.fmt == Q.MXFP4
    ef = helpers.unswizzle_scales(helpers.to_numpy_u8(qf.scales), 256, 512, 32).astype(np.int64)
    er = helpers.unswizzle_scales(helpers.to_numpy_u8(qr.scales), 256, 512, 32).astype(np.int64)
    d = er - ef
    assert set(np.unique(d).tolist()) == {0, 1}
    D = Q.gemm(qr, qr, torch.float32)
    torch.cuda.synchronize()
    Q.status()
    A = oracle_quant(x_dev.cpu(), Q.MXFP4_RU, Q.RTN, Q.HAD_NONE, Q.ROW)
    err = np.abs(D.cpu().numpy().astype(np.float64) - O.gemm(A, A))
    assert np.all(err <= O.gemm_bound(A, A))


def test_strided_input():
    """Row stride larger than the row (a column slice of a wider matrix)."""
    big = sweep_like(256, 512)
    x_dev = big.cuda()[:, 64:64 + 320]
    assert x_dev.stride(0) == 512
    for axis in (Q.ROW, Q.COL):
        for fmt in (Q.NVFP4, Q.MXFP4):
            q = gpu_quant(x_dev, fmt, Q.SR, Q.HAD_RAND16, axis)
            assert_same(q, oracle_quant(x_dev.cpu().contiguous(), fmt, Q.SR, Q.HAD_RAND16, axis), fmt)


def test_degenerate_inputs():
    for fmt in (Q.NVFP4, Q.MXFP4, Q.MXFP4_RU):
        for axis in (Q.ROW, Q.COL):
            z = torch.zeros((160, 96), dtype=torch.bfloat16)
            q = gpu_quant(z.cuda(), fmt, Q.QUARTET2, Q.HAD_RAND32, axis)
            assert_same(q, oracle_quant(z, fmt, Q.QUARTET2, Q.HAD_RAND32, axis), fmt)
            # huge and tiny magnitudes: saturation, E4M3 underflow to zero scales, subnormal E8M0 exponents
            x = torch.zeros((128, 128), dtype=torch.float32)
            x[0, 0] = 3.0e38
            x[1, :] = torch.linspace(-1e-30, 1e-30, 128)
            x[2, :] = 1e-38
            x[3, :7] = -2.5
            x = x.to(torch.bfloat16)
            for rnd in (Q.RTN, Q.SR, Q.QUARTET2):
                q = gpu_quant(x.cuda(), fmt, rnd, Q.HAD_NONE, axis)
                assert_same(q, oracle_quant(x, fmt, rnd, Q.HAD_NONE, axis), fmt)
            # empty tensors: nothing written but the tensor scale (1)
            e = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
            q = Q.quantize(e, fmt, Q.RTN, Q.HAD_NONE, axis)
            torch.cuda.synchronize()
            assert float(q.tensor_scale.cpu()[0]) == 1.0


def test_rtn_ties_and_grid():
    """Every E2M1 tie point and grid value, both signs, scaled into a block whose
    scale is exactly 1 (the block max is 6 and the tensor max maps to 6 * 448)."""
    vals = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0]
    row = torch.tensor(vals + [6.0], dtype=torch.float32)
    x = torch.cat([row, -row]).repeat(64, 1).reshape(64, 32).to(torch.bfloat16)
    for fmt in (Q.NVFP4, Q.MXFP4):
        q = gpu_quant(x.cuda(), fmt, Q.RTN, Q.HAD_NONE, Q.ROW)
        assert_same(q, oracle_quant(x, fmt, Q.RTN, Q.HAD_NONE, Q.ROW), fmt)


@pytest.mark.parametrize("axis", [Q.ROW, Q.COL])
@pytest.mark.parametrize("had", [Q.HAD_NONE, Q.HAD_DET32, Q.HAD_RAND16])
def test_amax_entry_point(axis, had):
    x = sweep_like(384, 256)
    seed = Q.make_seed(**SEED)
    a = Q.amax(x.cuda(), had, axis, seed)
    torch.cuda.synchronize()
    v = O.rotate(x, had, axis, SEED["rot"], SEED["rot_stream"])
    assert float(a.cpu()[0]) == float(np.abs(v).max())
    # the caller-provided amax path gives the same result as the internal pass
    q1 = gpu_quant(x.cuda(), Q.NVFP4, Q.RTN, had, axis, amax_in=a)
    assert_same(q1, oracle_quant(x, Q.NVFP4, Q.RTN, had, axis), Q.NVFP4)


@pytest.mark.parametrize("had", [Q.HAD_NONE, Q.HAD_DET16, Q.HAD_RAND16, Q.HAD_RAND32],
                         ids=["none", "det16", "rand16", "rand32"])
@pytest.mark.parametrize("shape", [(352, 416), (384, 256), (64, 128), (8192, 4096)], ids=lambda s: "x".join(map(str, s)))
def test_amax_rowcol_matches_oracle(had, shape):
    """Both orientations' amax from one call (one read of x for n_h <= 16, with
    different sign vectors per orientation) equal the oracle's max |rotated x|."""
    R, C = shape
    x = sweep_like(R, C)
    s_row = Q.make_seed(SEED["rot"], SEED["sr"], 1, 2)
    s_col = Q.make_seed(SEED["rot"], SEED["sr"], 2, 4)
    a = Q.amax_rowcol(x.cuda(), had, s_row, s_col).cpu().numpy()
    Q.status()
    v_row = O.rotate(x, had, O.ROW, SEED["rot"], 1)
    v_col = O.rotate(x, had, O.COL, SEED["rot"], 2)
    assert np.float32(a[0]) == np.float32(np.abs(v_row).max())
    assert np.float32(a[1]) == np.float32(np.abs(v_col).max())


@pytest.mark.parametrize("hads", [(Q.HAD_DET16, Q.HAD_RAND16), (Q.HAD_RAND16, Q.HAD_DET16), (Q.HAD_NONE, Q.HAD_RAND16),
                                  (Q.HAD_RAND32, Q.HAD_DET16)], ids=["det16-rand16", "rand16-det16", "none-rand16",
                                                                     "rand32-det16"])
@pytest.mark.parametrize("shape", [(352, 416), (384, 256), (8192, 4096)], ids=lambda s: "x".join(map(str, s)))
def test_amax_rowcol_with_a_hadamard_per_axis(hads, shape):
    """A Hadamard per orientation (the forward's deterministic one along K and
    the backward's random one along the tokens, as the linear layer uses them):
    one read of x when both have 16 points, one read per axis otherwise; each
    amax equals the oracle's max |rotated x| with that axis's Hadamard."""
    had_row, had_col = hads
    R, C = shape
    x = sweep_like(R, C)
    s_row = Q.make_seed(SEED["rot"], SEED["sr"], 0, 0)
    s_col = Q.make_seed(SEED["rot"], SEED["sr"], 2, 5)
    a = Q.amax_rowcol(x.cuda(), had_row, s_row, s_col, had_col=had_col).cpu().numpy()
    Q.status()
    v_row = O.rotate(x, had_row, O.ROW, SEED["rot"], 0)
    v_col = O.rotate(x, had_col, O.COL, SEED["rot"], 2)
    assert np.float32(a[0]) == np.float32(np.abs(v_row).max())
    assert np.float32(a[1]) == np.float32(np.abs(v_col).max())


def test_determinism_and_seed_sensitivity():
    x = sweep_like(256, 256).cuda()
    a = gpu_quant(x, Q.NVFP4, Q.SR, Q.HAD_RAND16, Q.COL)
    b = gpu_quant(x, Q.NVFP4, Q.SR, Q.HAD_RAND16, Q.COL)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
    c = Q.quantize(x, Q.NVFP4, Q.SR, Q.HAD_RAND16, Q.COL, Q.make_seed(1, 2, 3, 4))
    torch.cuda.synchronize()
    assert not torch.equal(a.codes, c.codes)


def test_argument_errors():
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Q.QFP4Error) as e:
        Q.quantize(x[:, :48], Q.MXFP4, Q.RTN, Q.HAD_NONE, Q.ROW)  # k = 48 not a multiple of 32
    assert e.value.status == Q.ERR_INVALID_ARG
    with pytest.raises(Q.QFP4Error) as e:
        Q.quantize(x[:, 1:33], Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW)  # 2-byte offset: misaligned
    assert e.value.status == Q.ERR_MISALIGNED
    with pytest.raises(Q.QFP4Error) as e:
        Q.quantize(x, Q.NVFP4, 9, Q.HAD_NONE, Q.ROW)
    assert e.value.status == Q.ERR_INVALID_ARG
    with pytest.raises(Q.QFP4Error) as e:
        Q.quantize(x, Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == Q.ERR_WORKSPACE
    Q.status()


@pytest.mark.parametrize("axis", [Q.ROW, Q.COL], ids=["row", "col"])
@pytest.mark.parametrize("had", [Q.HAD_NONE, Q.HAD_DET16, Q.HAD_RAND16], ids=["none", "det16", "rand16"])
@pytest.mark.parametrize("rnd", [Q.RTN, Q.QUARTET2], ids=["rtn", "q2"])
def test_fused_amax_matches_oracle(rnd, had, axis, monkeypatch):
    """With QFP4_FUSED_AMAX=1, NVFP4 tensors that fit in L2 are quantized by one
    cooperative launch that takes the rotated amax itself (a first pass, a grid
    barrier, then the quantizing pass); by default the separate amax pass runs
    instead (an amax launch, then the quantizer, which reduces the partials).
    Both give the oracle's codes, scales and tensor scale, on a shape with
    ragged tiles and on the full sweep tensor [8192 x 4096] (67 MB)."""
    for shape in ((384, 448), (8192, 4096)):
        x = sweep_like(*shape) if shape[0] < 8192 else inputs.workload("sweep")["T"]
        ref = oracle_quant(x, Q.NVFP4, rnd, had, axis)
        xd = x.cuda()
        monkeypatch.setenv("QFP4_FUSED_AMAX", "1")
        Q.launch_count(reset=True)
        assert_same(gpu_quant(xd, Q.NVFP4, rnd, had, axis), ref, Q.NVFP4)
        assert Q.launch_count(reset=True) == 1  # one cooperative launch
        monkeypatch.delenv("QFP4_FUSED_AMAX")
        assert_same(gpu_quant(xd, Q.NVFP4, rnd, had, axis), ref, Q.NVFP4)
        assert Q.launch_count(reset=True) == 2  # amax pass + quantizer
