"""Pins of the oracle's NVFP4 functions (no GPU).

NVFP4 as the LightX2V Wan2.2 checkpoint page describes it ("packed E2M1
weights with E4M3 block scales, plus FP32 input_global_scale and alpha
fields"), with the readings stated in oracle/mxfp8_oracle.c: 16-element
blocks, scale UE4M3(RN(amax * RN(g / 6))), elements E2M1(RN(x * RN(g /
dec(s)))), dequantized q dec(s) / g.

Independent checks: the E2M1 value set from the format's definition, a
brute-force nearest-value rounder written here, numpy binary32 arithmetic
and torch's E4M3 cast for the scales, and closed-form invariants.
"""
import numpy as np
import pytest
import torch

import oracle

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def brute_e2m1(v):
    """Nearest of the 8 magnitudes, ties to the even code; sign kept."""
    a = np.abs(v)
    d = np.abs(E2M1[None, :] - np.minimum(a, 6.0)[:, None])
    best = np.zeros(len(a), dtype=np.int64)
    for c in range(1, 8):
        better = (d[:, c] < d[np.arange(len(a)), best]) | ((d[:, c] == d[np.arange(len(a)), best]) & (c % 2 == 0))
        best = np.where(better, c, best)
    return (best | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def test_e2m1_table_from_the_format():
    vals = np.array([float(oracle.e2m1_decode(c)) for c in range(16)])
    assert np.array_equal(vals[:8], E2M1)
    assert np.array_equal(vals[8:], -E2M1) and np.all(np.signbit(vals[8:]))
    # sign bit 3, exponent bits 2-1 with bias 1, mantissa bit 0
    for c in range(1, 8):
        E, m = (c >> 1) & 3, c & 1
        assert vals[c] == (0.5 * m if E == 0 else 2.0 ** (E - 1) * (1 + 0.5 * m))


def test_e2m1_encode_ties_saturation_roundtrip():
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert int(oracle.e2m1_encode(v)) == c and int(oracle.e2m1_encode(-v)) == c | 8
    for v in (6.0, 6.5, 7.0, 100.0, 1e30):
        assert int(oracle.e2m1_encode(v)) == 7 and int(oracle.e2m1_encode(-v)) == 15
    for c in range(16):
        assert int(oracle.e2m1_encode(oracle.e2m1_decode(c))) == c
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-8, 8, 20000), rng.uniform(-1, 1, 20000)])
    assert np.array_equal(oracle.e2m1_encode(v), brute_e2m1(v))
    s = np.sort(rng.uniform(0, 7, 5000))
    dec = oracle.e2m1_decode(oracle.e2m1_encode(s))
    assert np.all(np.diff(dec) >= 0)


def _bits(x):
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _vals(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()


def _sample(seed, M=32, K=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, 3, replace=False)] *= 20
    bits = _bits(x)
    g = oracle.nvfp4_global_scale(np.abs(_vals(bits)).max())
    return bits, g


def test_scales_and_codes_follow_the_stated_binary32_steps():
    bits, g = _sample(1)
    q, s = oracle.nvfp4_quantize_bf16(bits, g)
    x = _vals(bits)
    M, K = x.shape
    blocks = x.reshape(M, K // 16, 16)
    gs = np.float32(g) / np.float32(6)
    sf = (np.abs(blocks).max(axis=2).astype(np.float32) * gs).astype(np.float32)
    expect_s = torch.from_numpy(sf).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, expect_s)
    ds = oracle.e4m3_decode(s).astype(np.float32)
    mul = np.where(ds > 0, np.float32(g) / np.where(ds > 0, ds, 1), 0).astype(np.float32)
    quot = (blocks * mul[:, :, None]).astype(np.float32).reshape(M, K)
    codes = brute_e2m1(quot.ravel().astype(np.float64)).reshape(M, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    assert np.array_equal(q, packed)


def test_low_nibble_holds_the_even_element():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0], x[0, 1] = 6.0, 1.0
    q, s = oracle.nvfp4_quantize_bf16(_bits(x), np.float32(1.0))
    assert s[0, 0] == 0x70 or oracle.e4m3_decode(s[0, 0]) == 1.0
    assert q[0, 0] == (7 | (2 << 4))


def test_largest_element_of_every_block_encodes_to_6():
    bits, g = _sample(2, M=64, K=512)
    q, s = oracle.nvfp4_quantize_bf16(bits, g)
    x = _vals(bits).reshape(64, 32, 16)
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(64, 32, 16)
    i = np.abs(x).argmax(axis=2)
    top = np.take_along_axis(codes, i[:, :, None], axis=2)[:, :, 0]
    normal = oracle.e4m3_decode(s) >= 2.0 ** -6          # scale in E4M3's normal range
    assert normal.mean() > 0.9
    assert np.all((top[normal] & 7) == 7)


def test_dequantize_and_error_bound():
    bits, g = _sample(3)
    q, s = oracle.nvfp4_quantize_bf16(bits, g)
    xhat = oracle.nvfp4_dequantize(q, s, g)
    x = _vals(bits).astype(np.float64)
    M, K = x.shape
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(M, K)
    ds = np.repeat(oracle.e4m3_decode(s), 16, axis=1)
    assert np.array_equal(xhat, oracle.e2m1_decode(codes) * ds / np.float64(np.float32(g)))
    # |x - xhat| <= half the E2M1 step at |x| g / dec(s), in x units, or the
    # saturation gap for the block maximum
    v = np.abs(x) * np.float64(np.float32(g)) / np.where(ds > 0, ds, np.inf)
    step = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))
    bound = np.maximum(step / 2, v - 6) * ds / np.float64(np.float32(g)) * (1 + 1e-6)
    assert np.all(np.abs(x - xhat) <= bound + 1e-30)


def test_linear_against_numpy():
    rng = np.random.default_rng(4)
    M, K, N = 7, 128, 9
    bx, gx = _sample(5, M=M, K=K)
    w = (rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32)
    bw = _bits(w)
    gw = oracle.nvfp4_global_scale(np.abs(_vals(bw)).max())
    xq, xs = oracle.nvfp4_quantize_bf16(bx, gx)
    wq, ws = oracle.nvfp4_quantize_bf16(bw, gw)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    y = oracle.nvfp4_linear(xq, xs, gx, wq, ws, gw, bias.view(np.uint16))
    ref = oracle.nvfp4_dequantize(xq, xs, gx) @ oracle.nvfp4_dequantize(wq, ws, gw).T + bias.astype(np.float64)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    ys = oracle.nvfp4_linear(xq, xs, gx, wq, ws, gw, bias.view(np.uint16), rows=[6, 1], cols=[8, 0, 3])
    assert np.array_equal(ys, y[[6, 1]][:, [8, 0, 3]])


def test_zero_block_gets_zero_scale_and_signed_zero_codes():
    x = np.ones((1, 32), dtype=np.float32)
    x[0, :16] = -0.0
    q, s = oracle.nvfp4_quantize_bf16(_bits(x), np.float32(448 * 6))
    assert s[0, 0] == 0 and np.all(q[0, :8] == 0x88)
    assert oracle.e4m3_decode(s[0, 1]) == 448


def test_global_scale_landmarks():
    """g = 448 * 6 / amax as a binary32 division (numpy's), which maps the
    tensor's largest block scale to 448 (the UE4M3 maximum); an all-zero,
    non-finite or underflowing amax gives 1."""
    for a in (1.0, 3.0, 0.1, 2688.0, 1e-30, 8e-36):
        want = np.float32(2688.0) / np.float32(a)
        assert oracle.nvfp4_global_scale(a) == want
        # the block holding amax gets the largest scale: amax g / 6 == 448
        assert abs(float(np.float32(a) * want / np.float32(6.0)) / 448.0 - 1.0) < 1e-6
    assert oracle.nvfp4_global_scale(0.0) == 1.0
    assert oracle.nvfp4_global_scale(float("inf")) == 1.0
    assert oracle.nvfp4_global_scale(float("nan")) == 1.0
    assert oracle.nvfp4_global_scale(1e-38) == 1.0          # 2688 / 1e-38 overflows binary32
