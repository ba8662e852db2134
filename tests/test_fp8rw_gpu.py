"""GPU parity of the per-channel FP8 path against the CPU oracle.

Quantizers: codes and FP32 scales bit-exact (both sides take the same
binary32 divisions, amax / 448 and x / s, and round the quotient to E4M3
nearest-even).  GEMM / layer: Y within |Y - Yref| <= 2^-7 |Yref| +
1e-3 rms(Yref) of the exact (FP64) oracle; the FP32 accumulation order is
not fixed.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_tol, bf16_bits, bf16_values, f16_bits
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    return mxfp8


@pytest.mark.parametrize("M,K", [(256, 512), (1, 8), (300, 5120), (129, 13824), (7, 16384), (1000, 1032)])
def test_activation_quantizer_bit_exact(mx, M, K):
    x = synth.activations_device(M, K, M + K, 0, "cuda")
    codes, scales = mx.fp8rw_quantize(x)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_rowwise_bf16(bf16_bits(x))
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_activation_quantizer_edge_rows(mx):
    M, K = 8, 1024
    x = synth.activations_device(M, K, 3, 0, "cuda")
    x[1] = 0.0
    x[2] = -0.0
    x[3] = 1e-38                                  # tiny: amax / 448 is subnormal
    x[4, 5] = 3.0e38                              # huge outlier
    x[5] = torch.linspace(-448, 448, K, device="cuda").to(torch.bfloat16)
    x[6] *= 2.0 ** -120
    codes, scales = mx.fp8rw_quantize(x)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_rowwise_bf16(bf16_bits(x))
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert scales[1].item() == 0.0 and int(codes[2, 0]) == 0x80


def test_activation_quantizer_strided_rows(mx):
    M, K = 200, 512
    big = synth.activations_device(M, 3 * K, 4, 0, "cuda")
    view = big[:, K: 2 * K]
    codes, scales = mx.fp8rw_quantize(view)
    c2, s2 = mx.fp8rw_quantize(view.contiguous())
    torch.cuda.synchronize()
    assert torch.equal(codes, c2) and torch.equal(scales, s2)


@pytest.mark.parametrize("N,K", [(512, 512), (5120, 5120), (333, 13824), (5, 4)])
def test_weight_quantizer_bit_exact(mx, N, K):
    w = synth.weights_device(N, K, N + K, 0, "cuda")
    codes, scales = mx.fp8rw_quantize_weight(w)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_rowwise_f32(w.cpu().numpy())
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def _layer(mx, M, K, N, seed, with_bias=True):
    x = synth.activations_device(M, K, seed, 0, "cuda")
    w = synth.weights_device(N, K, seed, 0, "cuda")
    b = synth.bias_device(N, seed, 0, "cuda") if with_bias else None
    wq, ws = mx.fp8rw_quantize_weight(w)
    return x, w, b, wq, ws


@pytest.mark.parametrize("M,K,N", [(256, 512, 512), (300, 512, 384), (1, 128, 8), (129, 256, 640),
                                   (1000, 1024, 1536), (517, 13824, 264)])
def test_linear_within_tolerance(mx, M, K, N):
    x, w, b, wq, ws = _layer(mx, M, K, N, seed=M + N)
    y = mx.fp8rw_linear(x, wq, ws, b)
    xq, xs = mx.fp8rw_quantize(x)
    y2 = mx.fp8rw_gemm(xq, xs, wq, ws, b)
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    assert torch.equal(y, y2), "fp8rw_linear differs from quantize + gemm"
    rq, rs = oracle.quantize_rowwise_bf16(bf16_bits(x))
    oq, os_ = oracle.quantize_rowwise_f32(w.cpu().numpy())
    yref = oracle.linear_rowwise(rq, rs, oq, os_, f16_bits(b))
    assert_within_tol(bf16_values(bf16_bits(y)), yref, f"fp8rw {M}x{K}x{N}")


def test_linear_without_bias_and_exact_integers(mx):
    # every row holds a 448 and small integers: the scale is exactly 1, the
    # codes are the integers, and the FP32 accumulation is exact (|sum| < 2^24),
    # so Y is the BF16 rounding of the exact integer result
    M, K, N = 130, 256, 136
    g = torch.Generator(device="cpu").manual_seed(5)
    xi = torch.randint(-8, 9, (M, K), generator=g).float()
    wi = torch.randint(-8, 9, (N, K), generator=g).float()
    xi[:, 0] = 448.0
    wi[:, 0] = -448.0
    x = xi.to(torch.bfloat16).cuda()
    wq, ws = mx.fp8rw_quantize_weight(wi.cuda())
    y = mx.fp8rw_linear(x, wq, ws, None)
    torch.cuda.synchronize()
    assert torch.all(ws == 1.0)
    exact = xi.double().numpy() @ wi.double().numpy().T
    assert np.array_equal(bf16_bits(y), oracle.bf16_rne(exact))


def test_q_projection_480p_full_size_sampled(mx):
    """M = 32760, K = N = 5120: all codes and scales bit-exact, sampled Y."""
    M, K, N, seed = synth.TOKENS_480P, synth.HIDDEN, synth.HIDDEN, 1
    x, w, b, wq, ws = _layer(mx, M, K, N, seed)
    xq, xs = mx.fp8rw_quantize(x)
    y = mx.fp8rw_gemm(xq, xs, wq, ws, b)
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    rq, rs = oracle.quantize_rowwise_bf16(bf16_bits(x))
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    oq, os_ = oracle.quantize_rowwise_f32(w.cpu().numpy())
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, M - 129, M - 1], np.arange(M - 40, M),
                                     rng.choice(M, 150, replace=False)]))
    cols = np.unique(np.concatenate([[0, 8, 255, 256, N - 1], rng.choice(N, 120, replace=False)]))
    yref = oracle.linear_rowwise(rq, rs, oq, os_, f16_bits(b), rows=rows, cols=cols)
    got = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
    assert_within_tol(bf16_values(bf16_bits(got)), yref, "fp8rw Q projection")


def test_single_cta_variant_in_subprocess():
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MXFP8_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(here, "test_fp8rw_gpu.py"), "-k", "linear_within or exact_integers"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
