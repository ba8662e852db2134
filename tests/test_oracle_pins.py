"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: a library
routine that implements the same format (PyTorch's float8_e4m3fn and
bfloat16 casts, numpy's float16), a closed form that the format or the rule
fixes, an invariant, or brute force on tiny inputs.  Together they are chosen
so that a plausible slip in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong rounding rule) fails at least one.

Passages: model card "Wan2.2-I2V-A14B-Lightning . MXFP8 (AutoRound OptRTN)",
SS "Quantization Details" (mx_fp, 8 bits, group_size 32, symmetric, dynamic
activations) and SS "Coverage per transformer" (E4M3 codes, per-32 E8M0
scales, F16 biases, about 13.99 GiB of quantized weights per transformer);
LightX2V "Model Quantization Techniques", Conv3D mode table (448 = E4M3 qmax
with FP32 accumulation).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_e4m3_decode(codes):
    t = torch.tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_e4m3_encode(values):
    # PyTorch's cast rounds to nearest even; it is not saturating (|v| >= 464
    # becomes NaN), so it is only a reference inside (-464, 464).
    t = torch.tensor(np.asarray(values, dtype=np.float64)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


ALL_CODES = np.arange(256, dtype=np.uint8)
FINITE_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
POS_FINITE = np.arange(0x7F, dtype=np.uint8)  # 0x00 .. 0x7E


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_all_256_codes_match_torch():
    ours = oracle.e4m3_decode(ALL_CODES)
    ref = torch_e4m3_decode(ALL_CODES)
    nan_o, nan_r = np.isnan(ours), np.isnan(ref)
    assert (nan_o == nan_r).all()
    assert np.array_equal(ours[~nan_o], ref[~nan_r])
    # sign symmetry including zero
    assert np.array_equal(np.abs(ours[:0x7F]), np.abs(ours[0x80:0xFF]))


def test_e4m3_landmarks_from_golden():
    # tests/golden/e4m3_landmarks.txt: code -> value, each line cites its source
    path = os.path.join(GOLDEN, "e4m3_landmarks.txt")
    n = 0
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        code_s, val_s = line.split()[:2]
        code = int(code_s, 16)
        val = oracle.e4m3_decode([code])[0]
        if val_s == "nan":
            assert math.isnan(val), line
        else:
            assert val == float.fromhex(val_s) if val_s.startswith(("0x", "-0x")) else val == float(val_s), line
        n += 1
    assert n >= 8


def test_e4m3_value_set_counts():
    vals = oracle.e4m3_decode(ALL_CODES)
    assert np.isnan(vals).sum() == 2                    # 0x7F, 0xFF
    finite = vals[~np.isnan(vals)]
    assert len(set(finite.tolist())) == 253             # +0 and -0 coincide
    assert finite.max() == 448.0 and finite.min() == -448.0
    pos = oracle.e4m3_decode(POS_FINITE)
    assert (np.diff(pos) > 0).all()                     # codes 0..0x7E increase


def test_e4m3_encode_roundtrip_all_finite_codes():
    vals = oracle.e4m3_decode(FINITE_CODES)
    # -0.0 must come back as 0x80: build the signed zero explicitly
    vals = np.where(FINITE_CODES == 0x80, -0.0, vals)
    assert np.array_equal(oracle.e4m3_encode(vals), FINITE_CODES)


def test_e4m3_encode_matches_torch_rne_inside_range():
    rng = np.random.default_rng(1234)
    pos = oracle.e4m3_decode(POS_FINITE)
    # PyTorch casts a float64 to float32 before it rounds to E4M3, so every
    # probe value is a float32 (exactly representable, no double rounding).
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)  # every tie
    near = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rand = np.concatenate([rng.uniform(-463.9, 463.9, 4000),
                           rng.standard_normal(4000) * 2.0 ** rng.integers(-12, 9, 4000)])
    rand = rand[np.abs(rand) < 463.9]
    v = np.concatenate([mids, -mids, near, -near, rand.astype(np.float32),
                        np.float32([448.0, 449.0, 463.99, -463.99])]).astype(np.float64)
    assert np.array_equal(oracle.e4m3_encode(v), torch_e4m3_encode(v))


def test_e4m3_ties_go_to_even_mantissa():
    # between 1.0 (0x38, mantissa 000) and 1.125 (0x39): the tie picks 0x38
    assert oracle.e4m3_encode([1.0625])[0] == 0x38
    # between 1.125 (0x39) and 1.25 (0x3A): the tie picks 0x3A
    assert oracle.e4m3_encode([1.1875])[0] == 0x3A
    # between the largest subnormal 7*2^-9 (0x07) and 2^-6 (0x08): picks 0x08
    assert oracle.e4m3_encode([7.5 * 2 ** -9])[0] == 0x08
    # between 0 and 2^-9: the tie picks +0 / -0
    assert oracle.e4m3_encode([2 ** -10])[0] == 0x00
    assert oracle.e4m3_encode([-(2 ** -10)])[0] == 0x80
    # between 416 (0x7D) and 448 (0x7E): picks 448 (mantissa 110 is even)
    assert oracle.e4m3_encode([432.0])[0] == 0x7E


def test_e4m3_encode_saturates_at_448():
    v = [448.0 * (1 + 2 ** -20), 463.99, 464.0, 480.0, 1e30, math.inf, -600.0, -1e30]
    assert oracle.e4m3_encode(v).tolist() == [0x7E] * 6 + [0xFE] * 2
    assert oracle.e4m3_encode([math.nan])[0] == 0x7F


def test_e4m3_encode_is_monotone():
    v = np.linspace(-500, 500, 200001)
    dec = oracle.e4m3_decode(oracle.e4m3_encode(v))
    assert (np.diff(dec) >= 0).all()


# ------------------------------------------------------------------ scale rule
@pytest.mark.parametrize("amax,byte", [
    (1.0, 119),              # floor(log2 1) = 0  -> e = -8
    (0.99, 118),             # floor(log2 .99) = -1
    (256.0, 127),            # e = 0
    (255.99, 126),
    (448.0, 127),
    (511.9, 127),
    (512.0, 128),
    (3.0, 120),
    (2.0 ** -118, 1),        # e = -126
    (2.0 ** -119, 0),        # e = -127, the E8M0 minimum
    (2.0 ** -133, 0),        # below the minimum: clamped
    (0.0, 0),                # all-zero block
    (2.0 ** 127, 246),       # e = 119
])
def test_scale_byte_landmarks(amax, byte):
    blk = np.zeros(32)
    blk[7] = amax
    blk[3] = -amax / 3
    _, s = oracle.quantize_block(blk)
    assert s == byte


def _half_ulp_e4m3(v):
    a = np.abs(v)
    ulp = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3))
    return ulp / 2


def test_block_invariants_random():
    rng = np.random.default_rng(7)
    for t in range(3000):
        mag = 2.0 ** rng.integers(-60, 60)
        blk = rng.standard_normal(32) * mag
        if t % 3 == 0:
            blk[rng.integers(0, 32)] *= 20.0            # an outlier
        if t % 7 == 0:
            blk[rng.integers(0, 32, 5)] = 0.0
        codes, s = oracle.quantize_block(blk)
        e = s - 127
        scale = 2.0 ** e
        amax = np.abs(blk).max()
        deq = oracle.e4m3_decode(codes) * scale
        assert 256 * scale <= amax < 512 * scale
        assert 256 * scale <= np.abs(deq).max() <= 448 * scale
        assert (np.abs(deq) <= 448 * scale).all()
        inside = np.abs(blk) < 448 * scale
        err = np.abs(deq - blk)
        assert (err[inside] <= _half_ulp_e4m3(blk[inside] / scale) * scale).all()
        assert (np.abs(deq[~inside]) == 448 * scale).all()
        assert (np.sign(deq[deq != 0]) == np.sign(blk[deq != 0])).all()


def test_block_lossless_when_exactly_representable():
    rng = np.random.default_rng(3)
    pos = oracle.e4m3_decode(POS_FINITE)
    top = np.where((pos >= 256) & (pos <= 448))[0]
    for _ in range(500):
        e = int(rng.integers(-100, 100))
        codes = rng.choice(FINITE_CODES, 32)
        codes[rng.integers(0, 32)] = rng.choice(top) | (0x80 if rng.random() < .5 else 0)
        codes = np.where(codes == 0x80, 0, codes).astype(np.uint8)  # no -0 inputs
        blk = oracle.e4m3_decode(codes) * 2.0 ** e
        got, s = oracle.quantize_block(blk)
        assert s == e + 127
        assert np.array_equal(got, codes)


def test_block_zero_and_signed_zero():
    codes, s = oracle.quantize_block(np.zeros(32))
    assert s == 0 and (codes == 0).all()
    codes, s = oracle.quantize_block(-np.zeros(32))
    assert s == 0 and (codes == 0x80).all()
    blk = np.zeros(32)
    blk[0], blk[1] = 1.0, -1e-6       # -1e-6 * 2^8 rounds to -0
    codes, s = oracle.quantize_block(blk)
    assert codes[1] == 0x80


def test_block_nonfinite():
    blk = np.ones(32)
    blk[5] = math.inf
    codes, s = oracle.quantize_block(blk)
    assert s == 0xFF and (codes == 0x7F).all()
    blk[5] = math.nan
    codes, s = oracle.quantize_block(blk)
    assert s == 0xFF and (codes == 0x7F).all()


def test_quantize_rows_match_blocks():
    rng = np.random.default_rng(11)
    x = torch.tensor(rng.standard_normal((3, 96)) * 5).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    codes, scales = oracle.quantize_bf16(bits)
    xd = x.to(torch.float64).numpy()
    for r in range(3):
        for b in range(3):
            c, s = oracle.quantize_block(xd[r, 32 * b:32 * b + 32])
            assert np.array_equal(codes[r, 32 * b:32 * b + 32], c) and scales[r, b] == s
    w = rng.standard_normal((4, 64)).astype(np.float32)
    codes, scales = oracle.quantize_f32(w)
    for r in range(4):
        for b in range(2):
            c, s = oracle.quantize_block(w[r, 32 * b:32 * b + 32].astype(np.float64))
            assert np.array_equal(codes[r, 32 * b:32 * b + 32], c) and scales[r, b] == s


# ------------------------------------------------------------------ BF16 / F16
def test_bf16_rne_matches_torch_on_float32_values():
    rng = np.random.default_rng(5)
    f = (rng.standard_normal(20000) * 2.0 ** rng.integers(-140, 120, 20000)).astype(np.float32)
    # exact ties: a BF16 value plus half of its ulp is a float32
    base = torch.tensor(f[:2000]).to(torch.bfloat16).to(torch.float32).numpy()
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    f = np.concatenate([f, ties, np.float32([0.0, -0.0, 1e-45, -3e38, 3.3e38])])
    ref = torch.tensor(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = oracle.bf16_rne(f.astype(np.float64))
    assert np.array_equal(ours, ref)


def test_bf16_decode_matches_torch():
    bits = np.arange(0, 65536, 7, dtype=np.uint16)
    ref = torch.tensor(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ours = oracle.bf16_decode(bits)
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.array_equal(ours[~both_nan], ref[~both_nan])


def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    ours = oracle.f16_decode(bits)
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert (np.isnan(ref) == np.isnan(ours)).all()
    assert np.array_equal(ours[~both_nan], ref[~both_nan])


# ------------------------------------------------------------------ linear
def _torch_dequant(codes, scales):
    v = torch_e4m3_decode(codes)
    s = np.repeat(2.0 ** (scales.astype(np.float64) - 127), 32, axis=1)
    return v * s


@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (3, 5, 64), (8, 7, 128), (2, 8, 96)])
def test_linear_exact_small_integers(M, N, K):
    # codes whose values are small integers, unit scales: every product and
    # sum is an exact integer, so the FP64 result must equal integer matmul.
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    ints = [c for c in range(256) if (c & 0x7F) != 0x7F
            and float(torch_e4m3_decode([c])[0]).is_integer()
            and abs(torch_e4m3_decode([c])[0]) <= 16]
    xq = rng.choice(ints, (M, K)).astype(np.uint8)
    wq = rng.choice(ints, (N, K)).astype(np.uint8)
    xs = np.full((M, K // 32), 127, np.uint8)
    ws = np.full((N, K // 32), 127, np.uint8)
    bias = rng.integers(-50, 50, N).astype(np.float16)
    xi = torch_e4m3_decode(xq).astype(np.int64)
    wi = torch_e4m3_decode(wq).astype(np.int64)
    expect = xi @ wi.T + bias.astype(np.int64)
    got = oracle.linear(xq, xs, wq, ws, bias.view(np.uint16))
    assert np.array_equal(got, expect.astype(np.float64))


def test_linear_block_scales_and_orientation_vs_numpy():
    rng = np.random.default_rng(99)
    M, N, K = 5, 7, 160
    xq = rng.choice(FINITE_CODES, (M, K)).astype(np.uint8)
    wq = rng.choice(FINITE_CODES, (N, K)).astype(np.uint8)
    xs = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)   # distinct per block
    ws = rng.integers(110, 140, (N, K // 32)).astype(np.uint8)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    expect = _torch_dequant(xq, xs) @ _torch_dequant(wq, ws).T + bias.astype(np.float64)
    got = oracle.linear(xq, xs, wq, ws, bias.view(np.uint16))
    assert np.allclose(got, expect, rtol=1e-12, atol=1e-12 * np.abs(expect).max())
    # no bias
    got0 = oracle.linear(xq, xs, wq, ws, None)
    assert np.allclose(got0, expect - bias.astype(np.float64), rtol=1e-12,
                       atol=1e-12 * np.abs(expect).max())


def test_linear_row_col_selection():
    rng = np.random.default_rng(17)
    M, N, K = 9, 11, 64
    xq = rng.choice(FINITE_CODES, (M, K)).astype(np.uint8)
    wq = rng.choice(FINITE_CODES, (N, K)).astype(np.uint8)
    xs = rng.integers(120, 135, (M, K // 32)).astype(np.uint8)
    ws = rng.integers(120, 135, (N, K // 32)).astype(np.uint8)
    full = oracle.linear(xq, xs, wq, ws)
    rows, cols = np.array([8, 0, 3]), np.array([10, 2])
    sub = oracle.linear(xq, xs, wq, ws, rows=rows, cols=cols)
    assert np.array_equal(sub, full[np.ix_(rows, cols)])


def test_dequantize_matches_torch():
    rng = np.random.default_rng(21)
    q = rng.choice(FINITE_CODES, (4, 96)).astype(np.uint8)
    s = rng.integers(100, 150, (4, 3)).astype(np.uint8)
    assert np.array_equal(oracle.dequantize(q, s), _torch_dequant(q, s))


# ------------------------------------------------------------------ GELU
def test_gelu_tanh_matches_torch_fp64():
    x = np.concatenate([np.linspace(-12, 12, 5001), [0.0, 1e-30, -1e-30, 50.0, -50.0]])
    ref = torch.nn.functional.gelu(torch.tensor(x), approximate="tanh").numpy()
    ours = oracle.gelu_tanh(x)
    # FP64 evaluation of the tanh form loses up to |x| 2^-53 to the
    # cancellation in 1 + tanh(u) for very negative x; the oracle avoids it.
    assert (np.abs(ours - ref) <= 1e-14 * np.abs(ref) + 2.0 ** -50 * np.abs(x)).all()
    # where there is no cancellation the two agree to rounding
    pos = x > -1
    assert np.allclose(ours[pos], ref[pos], rtol=1e-14, atol=0)


def test_gelu_tanh_closed_forms():
    assert oracle.gelu_tanh([0.0])[0] == 0.0
    x = np.linspace(0.01, 8, 400)
    # gelu(x) - gelu(-x) = x  (tanh is odd)
    assert np.allclose(oracle.gelu_tanh(x) - oracle.gelu_tanh(-x), x, rtol=1e-14)
    assert oracle.gelu_tanh([40.0])[0] == 40.0
    assert oracle.gelu_tanh([-40.0])[0] == 0.0


def test_gelu_bf16_is_rounded_fp64_gelu():
    rng = np.random.default_rng(2)
    x = torch.tensor(rng.standard_normal(3000) * 3).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    got = oracle.gelu_tanh_bf16(bits)
    ref_f64 = torch.nn.functional.gelu(x.to(torch.float64), approximate="tanh").numpy()
    # compare in value: the BF16 result is within half a BF16 ulp of the FP64 GELU
    got_v = torch.tensor(got.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref_f64), 2.0 ** -126))) - 7)
    xv = x.to(torch.float64).numpy()
    assert (np.abs(got_v - ref_f64) <= ulp / 2 * (1 + 1e-9) + 2.0 ** -49 * np.abs(xv)).all()


# ------------------------------------------------------------------ sizes
def test_weight_bytes_match_model_card_order_of_magnitude():
    # "The quantized weights are about 13.99 GiB per transformer" (model card,
    # Coverage per transformer): 40 blocks x 10 linears, 1 code byte per
    # weight plus 1 E8M0 byte per 32 weights.  Biases and packing metadata are
    # not counted here, so agreement to a few percent is all this pins.
    from mxfp8_w8a8_quantized_b200 import synth
    elems = 0
    for _, K, N, _ in synth.block_linears():
        elems += K * N
    elems *= synth.BLOCKS
    gib = (elems + elems // 32) / 2 ** 30
    assert abs(gib - 13.99) / 13.99 < 0.05, gib
    # 2-byte or 4-bit storage would miss by far
    assert abs(2 * elems / 2 ** 30 - 13.99) / 13.99 > 0.5


# ------------------------------------------------------------------ FP32 order
def test_linear_f32acc_is_sequential_float32_sum():
    # the FP32 evaluation is a left-to-right float32 accumulation of the exact
    # products: numpy's float32 add.accumulate computes the same sequence
    rng = np.random.default_rng(41)
    M, N, K = 3, 4, 96
    xq = rng.choice(FINITE_CODES, (M, K)).astype(np.uint8)
    wq = rng.choice(FINITE_CODES, (N, K)).astype(np.uint8)
    xs = rng.integers(118, 136, (M, K // 32)).astype(np.uint8)
    ws = rng.integers(118, 136, (N, K // 32)).astype(np.uint8)
    bias = (rng.standard_normal(N)).astype(np.float16)
    xd, wd = _torch_dequant(xq, xs), _torch_dequant(wq, ws)
    got = oracle.linear_f32acc(xq, xs, wq, ws, bias.view(np.uint16))
    for i in range(M):
        for j in range(N):
            prods = (xd[i] * wd[j]).astype(np.float32)
            assert np.array_equal(prods.astype(np.float64), xd[i] * wd[j])   # products exact
            s = np.add.accumulate(prods, dtype=np.float32)[-1]
            s = np.float32(s + np.float32(bias[j]))
            assert got[i, j] == float(s)


def test_linear_f32acc_within_float32_summation_bound():
    rng = np.random.default_rng(42)
    M, N, K = 4, 5, 512
    xq = rng.choice(FINITE_CODES, (M, K)).astype(np.uint8)
    wq = rng.choice(FINITE_CODES, (N, K)).astype(np.uint8)
    xs = rng.integers(115, 135, (M, K // 32)).astype(np.uint8)
    ws = rng.integers(115, 135, (N, K // 32)).astype(np.uint8)
    f64 = oracle.linear(xq, xs, wq, ws)
    f32 = oracle.linear_f32acc(xq, xs, wq, ws)
    absum = np.abs(_torch_dequant(xq, xs)) @ np.abs(_torch_dequant(wq, ws)).T
    assert (np.abs(f32 - f64) <= K * 2.0 ** -24 * absum).all()
    # integer-valued cases are exact in both
    ints = [c for c in range(256) if (c & 0x7F) != 0x7F and float(torch_e4m3_decode([c])[0]).is_integer()
            and abs(torch_e4m3_decode([c])[0]) <= 16]
    xq = rng.choice(ints, (M, K)).astype(np.uint8)
    wq = rng.choice(ints, (N, K)).astype(np.uint8)
    one = np.full((M, K // 32), 127, np.uint8)
    onew = np.full((N, K // 32), 127, np.uint8)
    assert np.array_equal(oracle.linear_f32acc(xq, one, wq, onew), oracle.linear(xq, one, wq, onew))
