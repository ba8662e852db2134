"""Failure detection on the GPU without a fault: each kernel family's bounded
wait is made to run out (one thread waits on an mbarrier that nothing arrives
at, with a 2 ms limit); the timeout must reach the host through
mxfp8_device_status() as MXFP8_ERR_TIMEOUT, be cleared by that read, and leave
the context usable (a layer computed afterwards still matches the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_tol, bf16_bits, bf16_values, f16_bits
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu

MXFP8_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def mx():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    return mxfp8


@pytest.mark.parametrize("which", [0, 1, 2])
def test_bounded_wait_reports_timeout_and_context_stays_usable(mx, which):
    assert mx.device_status() == 0
    mx.selftest_wait_timeout(which, 2_000_000)
    assert mx.device_status() == MXFP8_ERR_TIMEOUT
    assert mx.device_status() == 0, "the status read must clear the word"
    M, K, N = 256, 512, 512
    x = synth.activations_device(M, K, 11, 0, "cuda")
    w = synth.weights_device(N, K, 11, 0, "cuda")
    b = synth.bias_device(N, 11, 0, "cuda")
    wq, ws = mx.quantize_weight(w)
    y = mx.linear(x, wq, ws, b)
    assert mx.device_status() == 0
    xq, xs = oracle.quantize_bf16(bf16_bits(x))
    oq, os_ = oracle.quantize_f32(w.cpu().numpy())
    assert_within_tol(bf16_values(bf16_bits(y)), oracle.linear(xq, xs, oq, os_, f16_bits(b)),
                      "layer after a timed-out wait")
