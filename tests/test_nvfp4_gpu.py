"""GPU parity of the NVFP4 quantizers against the CPU oracle: packed E2M1
codes and UE4M3 scales bit-exact (both sides take the same binary32 steps),
tensor amax exact."""
import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_bits, bf16_values, unswizzle
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    return mxfp8


def _g(mx, t):
    amax = mx.nvfp4_amax(t).item()
    return mx.nvfp4_global_scale(amax), amax


@pytest.mark.parametrize("M,K", [(256, 512), (1, 16), (300, 5120), (129, 13824), (1000, 1040), (64, 48)])
def test_activation_quantizer_bit_exact(mx, M, K):
    x = synth.activations_device(M, K, M + K, 0, "cuda")
    g, amax = _g(mx, x)
    assert amax == float(np.abs(bf16_values(bf16_bits(x))).max())
    codes, scales = mx.nvfp4_quantize(x, g)
    torch.cuda.synchronize()
    rq, rs = oracle.nvfp4_quantize_bf16(bf16_bits(x), g)
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(unswizzle(scales.cpu().numpy(), M, K, 16), rs)


def test_activation_quantizer_edge_blocks_and_strides(mx):
    M, K = 8, 256
    big = synth.activations_device(M, 3 * K, 3, 0, "cuda")
    x = big[:, K: 2 * K]
    x[1] = 0.0
    x[2, :16] = -0.0
    x[3, 16:32] = 1e-30                         # scale underflows to 0 -> codes +-0
    x[4, 5] = 3.0e4                             # one huge element
    g = 448.0 * 6.0 / 3.0e4
    codes, scales = mx.nvfp4_quantize(x, g)
    torch.cuda.synchronize()
    rq, rs = oracle.nvfp4_quantize_bf16(bf16_bits(x), g)
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(unswizzle(scales.cpu().numpy(), M, K, 16), rs)
    c2, s2 = mx.nvfp4_quantize(x.contiguous(), g)
    torch.cuda.synchronize()
    assert torch.equal(codes, c2) and torch.equal(scales, s2)


@pytest.mark.parametrize("N,K", [(512, 512), (333, 13824), (8, 16)])
def test_weight_quantizer_rounds_to_bf16_first(mx, N, K):
    w = synth.weights_device(N, K, N + K, 0, "cuda")
    g, amax = _g(mx, w)
    wb = bf16_bits(w.to(torch.bfloat16))
    assert amax == float(np.abs(bf16_values(wb)).max())
    codes, scales = mx.nvfp4_quantize_weight(w, g)
    torch.cuda.synchronize()
    rq, rs = oracle.nvfp4_quantize_bf16(wb, g)
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(unswizzle(scales.cpu().numpy(), N, K, 16), rs)
