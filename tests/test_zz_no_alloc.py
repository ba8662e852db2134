"""mxfp8_linear_noalloc: the linear layer for callers that cannot allocate.

Some users of this library run inside another runtime's launch hook, where
allocating device memory is not allowed, or in a process whose allocator has
already reserved all of the GPU's memory, so a cudaMalloc (which also
synchronizes the whole device) would fail or stall other work.  They cannot
hand mxfp8_linear a workspace, so mxfp8_linear_noalloc quantizes into a fixed
scratch array that lives inside the library instead.

The entry point runs the same two kernels as mxfp8_linear on the same inputs,
only with its intermediate codes and scales in the library's scratch instead
of a caller workspace, so its output must equal mxfp8_linear's bit for bit.
The tests call it through the C-ABI twice in a row -- with different shapes,
the larger first, so that the second call also shows that whatever the first
one left in the shared scratch does not leak into its result -- and compare
each output with mxfp8_linear's (bit-identical) and with the CPU oracle
(within the tolerance the other GPU tests use).  A problem exactly at the
scratch's capacity is run the same way.  The file is collected after all the
others and passes both alone in a fresh process and after the rest of the
suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_tol, bf16_bits, bf16_values, f16_bits
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu

CODE_CAP = 32 << 20      # MXFP8_NOALLOC_MAX_CODE_BYTES


def _layer(M, K, N, seed):
    x = synth.activations(M, K, seed)
    w = synth.weights(N, K, seed)
    b = synth.bias(N, seed)
    return x, w, b


def _noalloc(mx, x, wq, ws, b):
    M, K = x.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    st = mx._lib.mxfp8_linear_noalloc(mx._ptr(x), M, K, mx._ptr(wq), mx._ptr(ws), N, mx._ptr(b),
                                      mx._ptr(y), mx._stream())
    assert st == 0, mx._lib.mxfp8_status_str(st)
    return y


def _oracle_rows(x, w, b, rows):
    """The oracle's FP64 linear on the given rows of X (weights quantized by
    the oracle from the same FP32 tensor)."""
    xb = bf16_bits(x[rows])
    xq, xs = oracle.quantize_bf16(xb)
    wq, ws = oracle.quantize_f32(w.numpy())
    return oracle.linear(xq, xs, wq, ws, f16_bits(b))


def _check(mx, cases, sample_rows=None):
    prepared = []
    for M, K, N, seed in cases:
        x, w, b = _layer(M, K, N, seed)
        wq, ws = mx.quantize_weight(w.cuda())
        prepared.append((x, w, b, x.cuda(), wq, ws, b.cuda()))
    outs = [_noalloc(mx, xd, wq, ws, bd) for _, _, _, xd, wq, ws, bd in prepared]   # back to back
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    for (x, w, b, xd, wq, ws, bd), y in zip(prepared, outs):
        ref = mx.linear(xd, wq, ws, bd)
        torch.cuda.synchronize()
        # same kernels, same inputs: only where the intermediate lives differs
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"noalloc != linear {tuple(x.shape)}"
        M = x.shape[0]
        rows = np.arange(M) if sample_rows is None else np.unique(np.r_[sample_rows(M), M - 1])
        yref = _oracle_rows(x, w, b, rows)
        assert_within_tol(bf16_values(bf16_bits(y))[rows], yref, f"noalloc vs oracle {tuple(x.shape)}")


def test_noalloc_matches_linear_and_oracle_on_two_calls_in_a_row():
    from mxfp8_w8a8_quantized_b200 import mxfp8 as mx
    # the larger problem first: the second call's scratch still holds its data
    cases = [(3000, 5120, 768, 31), (517, 1024, 264, 32)]
    _check(mx, cases, sample_rows=lambda M: np.arange(0, M, 7))


def test_noalloc_at_scratch_capacity():
    """M = floor(32 MiB / K) rows at K = 5120: the last code byte sits 5120
    bytes below the end of the codes region; then a small call reuses it."""
    from mxfp8_w8a8_quantized_b200 import mxfp8 as mx
    K = 5120
    M = CODE_CAP // K
    cases = [(M, K, 256, 33), (129, 256, 136, 34)]
    _check(mx, cases, sample_rows=lambda M: np.r_[np.arange(0, M, 97), np.arange(M - 40, M)])


def test_noalloc_rejects_problems_larger_than_its_scratch():
    from mxfp8_w8a8_quantized_b200 import mxfp8 as mx
    fake = ctypes.c_void_p(0x10000)
    K = 5120
    M = CODE_CAP // K + 1                          # one row more than the codes capacity
    st = mx._lib.mxfp8_linear_noalloc(fake, M, K, fake, fake, 256, None, fake, mx._stream())
    assert st == 3                                 # MXFP8_ERR_SHAPE, nothing launched
    K = (1 << 19) + 128                            # codes fit (16.8 MB), scales (2 MiB + 512 B) do not
    st = mx._lib.mxfp8_linear_noalloc(fake, 32, K, fake, fake, 256, None, fake, mx._stream())
    assert st == 3
