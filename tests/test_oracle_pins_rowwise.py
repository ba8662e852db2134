"""Pins of the oracle's per-channel FP8 functions against what the pages and
the mathematics fix (no GPU).

The scheme ("fp8-vllm" / "fp8-sgl" of "Model Quantization Techniques":
channel-symmetric FP8 weights, channel-dynamic symmetric FP8 activations,
scale = max(abs(x)) / qmax with qmax = 448 under FP32 accumulation; FP32
per-output-channel weight scales on the LightX2V FP8 checkpoint page):
  s = fp32(amax / 448),  q = E4M3_RNE_sat(fp32(x / s)),
  Y = s_x[m] s_w[n] sum_k q_x q_w + bias.
"""
import numpy as np
import pytest
import torch

import oracle


def _rows(seed, M=64, K=512, outliers=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    if outliers:
        ch = rng.choice(K, max(1, K // 100), replace=False)
        x[:, ch] *= 20
    # spread the rows over many binades
    x *= np.float32(2.0) ** rng.integers(-20, 20, size=(M, 1)).astype(np.float32)
    return x


def _bf16_bits(x):
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_vals(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()


def test_scale_is_fp32_amax_over_448():
    x = _rows(1)
    _, s = oracle.quantize_rowwise_f32(x)
    expect = np.abs(x).max(axis=1).astype(np.float32) / np.float32(448.0)
    assert s.dtype == np.float32 and np.array_equal(s, expect)


def test_codes_match_torch_e4m3_cast_of_fp32_quotient():
    # numpy's float32 division is the IEEE binary32 division; torch's cast of a
    # float32 to float8_e4m3fn rounds to nearest even (no saturation, but every
    # quotient here is at most 448 (1 + 2^-23), which rounds to 448)
    x = _rows(2)
    q, s = oracle.quantize_rowwise_f32(x)
    quot = x / s[:, None]
    assert np.abs(quot).max() < 449
    ref = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_largest_element_of_every_row_encodes_to_448():
    x = _rows(3)
    q, s = oracle.quantize_rowwise_f32(x)
    i = np.abs(x).argmax(axis=1)
    top = q[np.arange(len(x)), i]
    sign = np.signbit(x[np.arange(len(x)), i])
    assert np.all(top == np.where(sign, 0xFE, 0x7E))
    # and no code exceeds it
    dec = oracle.e4m3_decode(q)
    assert np.abs(dec).max() <= 448


def test_elementwise_error_is_half_an_e4m3_step():
    x = _rows(4)
    q, s = oracle.quantize_rowwise_f32(x)
    xr = x.astype(np.float64) / s[:, None].astype(np.float64)
    dec = oracle.e4m3_decode(q)
    a = np.abs(xr)
    # E4M3 spacing at |v|: 2^(floor(log2 v) - 3) for v >= 2^-6, else 2^-9
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    half = np.ldexp(1.0, (e - 4).astype(int))
    # the binary32 quotient adds at most one float32 ulp of |v| on top
    assert np.all(np.abs(dec - xr) <= half + a * 2.0 ** -23)


def test_zero_row_and_signed_zero():
    x = _rows(5, M=4)
    x[1] = 0.0
    x[2] = -0.0
    q, s = oracle.quantize_rowwise_f32(x)
    assert s[1] == 0 and s[2] == 0
    assert np.all(q[1] == 0x00) and np.all(q[2] == 0x80)


def test_bf16_activation_path_equals_f32_path_on_the_same_values():
    x = _rows(6)
    bits = _bf16_bits(x)
    qa, sa = oracle.quantize_rowwise_bf16(bits)
    qb, sb = oracle.quantize_rowwise_f32(_bf16_vals(bits))
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb)


def test_linear_rowwise_against_numpy():
    rng = np.random.default_rng(7)
    M, K, N = 9, 96, 13          # M != N: swapped scale vectors would not even fit
    x = _rows(8, M=M, K=K)
    w = rng.standard_normal((N, K)).astype(np.float32) / np.sqrt(K)
    xq, sx = oracle.quantize_rowwise_f32(x)
    wq, sw = oracle.quantize_rowwise_f32(w)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    y = oracle.linear_rowwise(xq, sx, wq, sw, bias.view(np.uint16))
    xd = oracle.e4m3_decode(xq) * sx[:, None].astype(np.float64)
    wd = oracle.e4m3_decode(wq) * sw[:, None].astype(np.float64)
    ref = xd @ wd.T + bias.astype(np.float64)[None, :]
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # row / column selection
    ys = oracle.linear_rowwise(xq, sx, wq, sw, bias.view(np.uint16), rows=[8, 0, 3], cols=[12, 1])
    assert np.array_equal(ys, y[[8, 0, 3]][:, [12, 1]])


def test_linear_rowwise_exact_small_integers():
    # codes of small integers with power-of-two scales: every step is exact
    M, K, N = 3, 64, 5
    rng = np.random.default_rng(9)
    xi = rng.integers(-8, 9, size=(M, K)).astype(np.float64)
    wi = rng.integers(-8, 9, size=(N, K)).astype(np.float64)
    xq = oracle.e4m3_encode(xi)
    wq = oracle.e4m3_encode(wi)
    sx = (2.0 ** rng.integers(-4, 4, size=M)).astype(np.float32)
    sw = (2.0 ** rng.integers(-4, 4, size=N)).astype(np.float32)
    y = oracle.linear_rowwise(xq, sx, wq, sw)
    ref = (xi @ wi.T) * sx[:, None] * sw[None, :]
    assert np.array_equal(y, ref)
