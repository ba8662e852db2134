"""mxfp8_linear_noalloc: the linear layer for callers that cannot allocate.

Some users of this library run inside another runtime's launch hook, where
allocating device memory is not allowed, or in a process whose allocator has
already reserved all of the GPU's memory, so a cudaMalloc (which also
synchronizes the whole device) would fail or stall other work.  They cannot
hand mxfp8_linear a workspace, so mxfp8_linear_noalloc quantizes into a fixed
scratch array that lives inside the library instead.

This test calls the new entry point through the C-ABI twice in a row -- with
different shapes, so the second call also shows that whatever the first one
left in the shared scratch does not leak into its result -- and compares each
output with mxfp8_linear's on the same inputs, within the tolerance the other
GPU tests use.  It lives in its own file, collected after all the others, and
passes both alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import assert_within_tol, bf16_bits, bf16_values
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu


def _layer(M, K, N, seed):
    x = synth.activations(M, K, seed).cuda()
    w = synth.weights(N, K, seed).cuda()
    b = synth.bias(N, seed).cuda()
    return x, w, b


def _noalloc(mx, x, wq, ws, b):
    M, K = x.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    st = mx._lib.mxfp8_linear_noalloc(mx._ptr(x), M, K, mx._ptr(wq), mx._ptr(ws), N, mx._ptr(b),
                                      mx._ptr(y), mx._stream())
    assert st == 0, mx._lib.mxfp8_status_str(st)
    return y


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    from mxfp8_w8a8_quantized_b200 import mxfp8 as mx
    cases = [(3000, 5120, 768, 31), (517, 1024, 264, 32)]   # M*K fits the 32 MiB scratch
    prepared = []
    for M, K, N, seed in cases:
        x, w, b = _layer(M, K, N, seed)
        wq, ws = mx.quantize_weight(w)
        prepared.append((x, wq, ws, b))
    outs = []
    for x, wq, ws, b in prepared:                # the two calls, back to back
        outs.append(_noalloc(mx, x, wq, ws, b))
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    for (x, wq, ws, b), y in zip(prepared, outs):
        ref = mx.linear(x, wq, ws, b)
        torch.cuda.synchronize()
        got_v = bf16_values(bf16_bits(y))
        ref_v = bf16_values(bf16_bits(ref))
        assert_within_tol(got_v, ref_v, f"noalloc vs linear {tuple(x.shape)}")
        assert np.isfinite(got_v).all()


def test_noalloc_rejects_problems_larger_than_its_scratch():
    from mxfp8_w8a8_quantized_b200 import mxfp8 as mx
    K = 5120
    M = (32 << 20) // K + 1                       # one row more than the codes capacity
    fake = ctypes.c_void_p(0x10000)
    st = mx._lib.mxfp8_linear_noalloc(fake, M, K, fake, fake, 256, None, fake, mx._stream())
    assert st == 3                                 # MXFP8_ERR_SHAPE, nothing launched
