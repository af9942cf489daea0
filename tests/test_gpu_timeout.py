"""GPU: the timeout path of the bounded waits, made to run out without a fault.

The test hook qlinear_debug_gemv_stalled holds back the GEMV's weight copies,
so every consumer's bounded wait gives up after about 2 s.  The kernel must
record QL_ERR_TIMEOUT with its kernel id and wait site in the status word and
return; the status read clears it, and the same context then computes a
correct product.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu

KID_GEMV, SITE_CONSUMER_FULL = 1, 2


def test_gemv_wait_timeout_is_recorded_and_context_survives(cuda):
    scheme, N, K = ql.FP8_E4M3_ROW, 1024, 4096
    x = synthetic.make_x(1, K, seed=9, tag="timeout-x", outliers=3)
    w = synthetic.make_w(N, K, seed=9, tag="timeout-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    dx, dwq, dsw = bf16_dev(x), u8_dev(wq), f32_dev(sw)
    assert ql.device_status()[0] == 0
    ql.debug_gemv_stalled(scheme, dx, dwq, dsw)
    st, detail = ql.device_status()
    assert st == 5, ql.lib().qlinear_status_string(st)  # QL_ERR_TIMEOUT
    assert detail == (KID_GEMV << 8) | SITE_CONSUMER_FULL
    assert ql.device_status() == (0, 0)  # read-and-clear
    y = ql.gemv(scheme, dx, dwq, dsw)
    assert ql.device_status()[0] == 0
    assert_y_close(bits(y), oracle.forward(scheme, x, wq, sw), "gemv after a timeout")
