"""The oracle's row-subset quantization (used to check full-size GPU results
on sampled rows) gives exactly the rows the whole-tensor quantization gives:
the same tensor amax, the same random words (those of each row's own index),
for every format, rounding and orientation."""
import numpy as np
import pytest

import oracle as O
from fp4_precision_b200 import inputs


@pytest.mark.parametrize("axis", [O.ROW, O.COL], ids=["row", "col"])
@pytest.mark.parametrize("fmt,rnd,had", [(O.NVFP4, O.SR, O.HAD_RAND16), (O.NVFP4, O.QUARTET2, O.HAD_RAND16),
                                         (O.MXFP4, O.QUARTET2, O.HAD_DET32), (O.MXFP4_RU, O.SR, O.HAD_NONE),
                                         (O.NVFP4, O.RTN, O.HAD_NONE)])
def test_row_subset_equals_whole_tensor_rows(fmt, rnd, had, axis):
    x = inputs.student_t_colgain((192, 256), 3, "subset")
    full = O.quantize(x, fmt, rnd, had, axis, 11, 2, 13, 5)
    sel = np.array([full.rows - 1, 0, 17, 17, 64, 3])
    sub = O.quantize(x, fmt, rnd, had, axis, 11, 2, 13, 5, rows_sel=sel)
    assert sub.rows == len(sel) and sub.g == full.g
    assert np.array_equal(sub.codes, full.codes[sel])
    assert np.array_equal(sub.scales, full.scales[sel])
    assert np.array_equal(sub.alpha, full.alpha[sel])


def test_row_subset_rejects_out_of_range():
    x = inputs.normal((64, 64), 1.0, 1, "r")
    with pytest.raises(ValueError):
        O.quantize(x, O.NVFP4, O.RTN, O.HAD_NONE, O.ROW, rows_sel=[64])
