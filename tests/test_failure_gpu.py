"""Failure detection on the GPU without a fault: a kernel whose wait nothing
satisfies gives up after the library's wait limit, reports MXFP4_ERR_TIMEOUT
through the device status word, and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import _lib
from helpers import bits_of

pytestmark = pytest.mark.gpu


def test_stalled_wait_reports_timeout_and_context_survives():
    assert mx.mxfp4_get_device_status() == _lib.OK          # clean slate
    t0 = time.perf_counter()
    mx.mxfp4_selftest_wait_timeout()
    status = mx.mxfp4_get_device_status()                   # synchronizes
    waited = time.perf_counter() - t0
    assert status == _lib.ERR_TIMEOUT
    assert 1.5 < waited < 30.0                               # the 2 s wait limit, not a hang
    assert mx.mxfp4_get_device_status() == _lib.OK          # reading clears the word
    # the context still works: a quantize afterwards is bit-exact
    g = torch.Generator().manual_seed(9)
    x = torch.randn(64, 256, generator=g).to(torch.bfloat16)
    codes, scales = mx.mxfp4_quantize(x.cuda())
    rc, rs = oracle.quantize(bits_of(x))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert mx.mxfp4_get_device_status() == _lib.OK
