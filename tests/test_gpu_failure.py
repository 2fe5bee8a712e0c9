"""Failure detection without a GPU fault: every wait in the library's kernels
is bounded; when one runs out the kernel sets the device error word and
returns, qfp4_status reports QFP4_ERR_TIMEOUT and clears it, and the context
stays usable. The wait here is on a shared-memory barrier nothing arrives on,
with a 50 ms limit."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

pytestmark = pytest.mark.gpu


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_bounded_wait_reports_timeout_and_the_context_stays_usable():
    Q.status()  # nothing pending
    assert Q.lib().qfp4_selftest_wait_timeout(50_000_000, _stream()) == Q.OK
    with pytest.raises(Q.QFP4Error) as e:
        Q.status()
    assert e.value.status == Q.ERR_TIMEOUT
    Q.status()  # the error word was cleared
    # the library still works after the timeout: a quantization matches the oracle
    x = inputs.normal((256, 512), 1.0, 41, "after_timeout")
    q = Q.quantize(x.cuda(), Q.NVFP4, Q.RTN, Q.HAD_DET16, Q.ROW, Q.make_seed())
    Q.status()
    ref = O.quantize(x, O.NVFP4, O.RTN, O.HAD_DET16, O.ROW)
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes)


def test_selftest_rejects_limits_outside_the_bound():
    for bad in (0, -1, 3_000_000_000):
        assert Q.lib().qfp4_selftest_wait_timeout(bad, _stream()) == Q.ERR_INVALID_ARG
