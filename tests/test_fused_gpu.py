"""The GEMM whose epilogue quantizes for the next linear
(mxfp8_gemm_quantize_out), with and without GELU.

1. Bit for bit against the separate kernels on the same inputs:
   gemm_prequant -> [gelu_tanh] -> quantize writes the same codes and the
   same scale bytes (padding included) as the fused launch.
2. Against the oracle's chain (exact linear -> BF16 -> [GELU -> BF16] ->
   quantize): the BF16 value a code is taken from may differ in its last bit
   (the FP32 summation order is open), which moves a code by at most one E4M3
   step, and only rarely (a BF16 ulp is 1/32 of an E4M3 step); so at most
   1e-3 of the codes may differ, each by at most one step of its block.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_bits, f16_bits, unswizzle
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5


@pytest.fixture(scope="module")
def mx():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    return mxfp8


def layer(mx, M, K, N, seed, with_bias=True):
    x = synth.activations_device(M, K, seed, 0, "cuda")
    w = synth.weights_device(N, K, seed, 0, "cuda")
    b = synth.bias_device(N, seed, 0, "cuda") if with_bias else None
    wq, ws = mx.quantize_weight(w)
    xq, xs = mx.quantize(x)
    return x, w, b, wq, ws, xq, xs


def filled(n, dev="cuda"):
    return torch.full((n,), SENTINEL, dtype=torch.uint8, device=dev)


def fused(mx, xq, xs, wq, ws, b, act, M, N):
    codes = filled(M * N + 64)
    scales = filled(mx.scale_bytes(M, N) + 64)
    mx.gemm_quantize_out(xq, xs, wq, ws, b, act=act, codes=codes[: M * N].view(M, N),
                         scales=scales[: mx.scale_bytes(M, N)])
    return codes, scales


def separate(mx, xq, xs, wq, ws, b, act, M, N):
    y = mx.gemm_prequant(xq, xs, wq, ws, b)
    if act == mx.ACT_GELU_TANH:
        mx.gelu_tanh(y, out=y)
    codes = filled(M * N + 64)
    scales = filled(mx.scale_bytes(M, N) + 64)
    mx.quantize(y, codes=codes[: M * N].view(M, N), scales=scales[: mx.scale_bytes(M, N)])
    return codes, scales, y


SHAPES = [
    (256, 512, 512),      # the small single-linear case
    (300, 512, 384),      # ragged M, N = 1.5 tiles (half a tile's warps idle)
    (1, 128, 128),        # one row, one K step
    (129, 256, 640),      # one row past a tile, 2.5 N tiles
    (1000, 1024, 1536),
    (4097, 512, 256),     # many M tiles, ragged by one row
    (200, 13824, 256),    # long K (ffn.net.2's)
    (384, 256, 13824),    # wide N (ffn.net.0.proj's)
]


@pytest.mark.parametrize("M,K,N", SHAPES)
@pytest.mark.parametrize("gelu", [False, True])
def test_fused_equals_separate_kernels(mx, M, K, N, gelu):
    x, w, b, wq, ws, xq, xs = layer(mx, M, K, N, seed=M + K + N)
    act = mx.ACT_GELU_TANH if gelu else mx.ACT_NONE
    cf, sf = fused(mx, xq, xs, wq, ws, b, act, M, N)
    cs, ss, _ = separate(mx, xq, xs, wq, ws, b, act, M, N)
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    assert torch.equal(cf, cs), "codes differ from GEMM -> [GELU] -> quantize"
    assert torch.equal(sf, ss), "scale bytes (or their padding) differ"
    assert int(cf[M * N:].ne(SENTINEL).sum()) == 0, "wrote past the codes"
    assert int(sf[mx.scale_bytes(M, N):].ne(SENTINEL).sum()) == 0, "wrote past the scales"


def test_fused_without_bias(mx):
    M, K, N = 300, 512, 384
    x, w, b, wq, ws, xq, xs = layer(mx, M, K, N, seed=5, with_bias=False)
    cf, sf = fused(mx, xq, xs, wq, ws, None, mx.ACT_GELU_TANH, M, N)
    cs, ss, _ = separate(mx, xq, xs, wq, ws, None, mx.ACT_GELU_TANH, M, N)
    torch.cuda.synchronize()
    assert torch.equal(cf, cs) and torch.equal(sf, ss)


def _e4m3_step(scale_bytes):
    """One E4M3 step at the top binade of each block, as a value: the
    coarsest spacing any code of the block can have (2^-3 * 2^8 * 2^e)."""
    return np.ldexp(1.0, scale_bytes.astype(np.int64) - 127 + 5)


@pytest.mark.parametrize("gelu", [False, True])
def test_fused_against_oracle_chain(mx, gelu):
    M, K, N = 300, 1024, 640
    seed = 11
    x, w, b, wq, ws, xq, xs = layer(mx, M, K, N, seed)
    act = mx.ACT_GELU_TANH if gelu else mx.ACT_NONE
    cf, sf = fused(mx, xq, xs, wq, ws, b, act, M, N)
    torch.cuda.synchronize()
    got_c = cf[: M * N].view(M, N).cpu().numpy()
    got_s = unswizzle(sf[: mx.scale_bytes(M, N)].cpu().numpy(), M, N)

    rq, rs = oracle.quantize_bf16(bf16_bits(x))
    oq, os_ = oracle.quantize_f32(w.cpu().numpy())
    y = oracle.bf16_rne(oracle.linear(rq, rs, oq, os_, f16_bits(b)))
    if gelu:
        y = oracle.gelu_tanh_bf16(y)
    ref_c, ref_s = oracle.quantize_bf16(y)

    got = oracle.dequantize(got_c, got_s)
    ref = oracle.dequantize(ref_c, ref_s)
    differ = got_c != ref_c
    assert differ.mean() <= 1e-3, f"{differ.mean():.2e} of codes differ"
    step = np.repeat(_e4m3_step(np.maximum(got_s, ref_s)), 32, axis=1)
    assert np.all(np.abs(got - ref) <= step), "a code moved by more than one E4M3 step"
    assert (got_s != ref_s).mean() <= 1e-2


def test_fused_argument_errors(mx):
    M, K, N = 128, 256, 256
    x, w, b, wq, ws, xq, xs = layer(mx, M, K, N, seed=3)
    with pytest.raises(mx.MXFP8Error) as e:
        mx.gemm_quantize_out(xq, xs, wq, ws, b, act=7)
    assert e.value.status == 1                       # unknown activation
    # N must be a multiple of 128 (the next linear's K)
    w2 = synth.weights_device(200, K, 3, 1, "cuda")
    wq2, ws2 = mx.quantize_weight(w2)
    with pytest.raises(mx.MXFP8Error) as e:
        mx.gemm_quantize_out(xq, xs, wq2, ws2, None)
    assert e.value.status == 3
    # M = 0 launches nothing and succeeds
    codes = torch.empty((0, N), dtype=torch.uint8, device="cuda")
    mx.gemm_quantize_out(xq[:0], xs, wq, ws, b, codes=codes, scales=torch.empty(16, dtype=torch.uint8,
                                                                                    device="cuda"))
    torch.cuda.synchronize()
    assert mx.device_status() == 0


def test_fused_repeatable(mx):
    M, K, N = 1000, 1024, 1536
    x, w, b, wq, ws, xq, xs = layer(mx, M, K, N, seed=9)
    c1, s1 = fused(mx, xq, xs, wq, ws, b, mx.ACT_GELU_TANH, M, N)
    c2, s2 = fused(mx, xq, xs, wq, ws, b, mx.ACT_GELU_TANH, M, N)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


def test_fused_single_cta_variant_in_subprocess():
    # the CTA-pair variant is the default; the single-CTA one is fixed per
    # process, so it is checked in a child
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MXFP8_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(here, "test_fused_gpu.py"), "-k", "equals_separate"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
