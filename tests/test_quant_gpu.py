"""GPU parity of the MX quantizer kernels against the CPU oracle: codes and
scales must match bit for bit, in both scale layouts, on the workload
distribution, ragged shapes and adversarial blocks."""
import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_bits, tc_bytes, tc_index, unswizzle
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    return mxfp8


def gpu_quant(mx, x_cpu_bf16, layout):
    x = x_cpu_bf16.cuda()
    codes, scales = mx.quantize(x, layout=layout)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def check_act(mx, x_cpu, what):
    M, K = x_cpu.shape
    ref_c, ref_s = oracle.quantize_bf16(bf16_bits(x_cpu))
    c, s = gpu_quant(mx, x_cpu, mx.SF_ROWMAJOR)
    assert np.array_equal(c, ref_c), f"{what}: codes differ at {np.argwhere(c != ref_c)[:5].tolist()}"
    assert np.array_equal(s.reshape(M, K // 32), ref_s), f"{what}: row-major scales differ"
    c2, s2 = gpu_quant(mx, x_cpu, mx.SF_TCGEN05)
    assert np.array_equal(c2, ref_c)
    assert s2.size == tc_bytes(M, K)
    assert np.array_equal(unswizzle(s2, M, K), ref_s), f"{what}: tensor-core scales differ"
    # every byte not addressed by a real (row, block) is padding and must be 0
    used = np.zeros(s2.size, bool)
    used[tc_index(M, K).ravel()] = True
    assert (s2[~used] == 0).all(), f"{what}: padding not zero"


# (40000, 96): more rows than the quantizer's resident warps (32 x 148
# blocks x 8), so warps walk a second row; one partial segment per row.
@pytest.mark.parametrize("M,K", [(256, 512), (1, 32), (7, 96), (129, 256), (300, 160), (128, 5120),
                                 (37, 13824), (1000, 640), (40000, 96)])
def test_activation_quant_workload_distribution(mx, M, K):
    x = synth.activations(M, K, seed=M + K)
    check_act(mx, x, f"M={M} K={K}")


def adversarial_rows(K=256):
    """Rows of blocks that probe every corner of the rule."""
    rows = []
    z = np.zeros(K, np.float32)
    rows.append(z.copy())                                  # all-zero blocks
    rows.append(-z)                                        # -0 everywhere
    r = np.zeros(K, np.float32)
    r[0::32] = 1.0                                         # amax exactly a power of two
    r[1::32] = -(1.0 + 2 ** -7)                            # near-tie values
    rows.append(r)
    # exact E4M3 midpoints (ties) after scaling by 2^-e with amax = 256 * 2^e
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2)
    r = np.zeros(K, np.float32)
    for b in range(K // 32):
        r[32 * b] = 256.0
        r[32 * b + 1: 32 * b + 32] = mids[(np.arange(31) + 31 * b) % len(mids)]
    rows.append(r * 2.0 ** -3)
    # values in (448, 512) * 2^e that saturate
    r = np.zeros(K, np.float32)
    for b in range(K // 32):
        r[32 * b: 32 * b + 32] = np.linspace(300, 511, 32) * (1 if b % 2 else -1)
    rows.append(r)
    # subnormal-range blocks (BF16 subnormals and tiny normals)
    r = np.zeros(K, np.float32)
    r[:64] = np.float32(2.0 ** -130) * np.arange(64)
    r[64:128] = np.float32(2.0 ** -120) * np.linspace(-3, 3, 64)
    r[128:] = np.float32(2.0 ** 120) * np.linspace(-1, 1, K - 128)
    rows.append(r)
    # huge magnitudes up to the BF16 maximum
    r = np.full(K, 3.0e38, np.float32)
    r[1::2] = -1.0
    rows.append(r)
    return torch.tensor(np.stack(rows)).to(torch.bfloat16)


def test_activation_quant_adversarial_blocks(mx):
    x = adversarial_rows()
    check_act(mx, x, "adversarial")


def test_activation_quant_nonfinite_blocks(mx):
    x = torch.randn(4, 128).to(torch.bfloat16)
    x[0, 5] = float("inf")
    x[1, 40] = float("nan")
    x[2, 100] = float("-inf")
    check_act(mx, x, "non-finite")


def test_activation_quant_strided_input(mx):
    x_full = synth.activations(64, 1024, seed=5)
    x = x_full.cuda()[:, :512]             # row stride 1024 elements
    ref_c, ref_s = oracle.quantize_bf16(bf16_bits(x_full[:, :512]))
    codes = torch.empty((64, 512), dtype=torch.uint8, device="cuda")
    scales = torch.empty(64 * 16, dtype=torch.uint8, device="cuda")
    st = mx._lib.mxfp8_quantize(mx._ptr(x), 64, 512, 1024, mx._ptr(codes), mx._ptr(scales),
                                mx.SF_ROWMAJOR, mx._stream())
    assert st == 0
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), ref_c)
    assert np.array_equal(scales.cpu().numpy().reshape(64, 16), ref_s)


@pytest.mark.parametrize("N,K", [(512, 512), (8, 32), (264, 384), (1, 13824)])
def test_weight_quant_fp32(mx, N, K):
    w = synth.weights(N, K, seed=N)
    w[0, :32] = 0.0
    if N > 1:
        w[1, :32] = torch.linspace(-600, 600, 32)
    ref_c, ref_s = oracle.quantize_f32(w.numpy())
    c, s = mx.quantize_weight(w.cuda(), layout=mx.SF_ROWMAJOR)
    assert np.array_equal(c.cpu().numpy(), ref_c)
    assert np.array_equal(s.cpu().numpy().reshape(N, K // 32), ref_s)
    c2, s2 = mx.quantize_weight(w.cuda(), layout=mx.SF_TCGEN05)
    assert np.array_equal(c2.cpu().numpy(), ref_c)
    assert np.array_equal(unswizzle(s2.cpu().numpy(), N, K), ref_s)


def test_weight_quant_fp32_tiny_and_subnormal(mx):
    w = torch.zeros(3, 64)
    w[0] = torch.linspace(-1e-38, 1e-38, 64)   # FP32 subnormals
    w[1] = torch.linspace(-3e38, 3e38, 64)
    w[2, ::3] = 2.0 ** -126
    ref_c, ref_s = oracle.quantize_f32(w.numpy())
    c, s = mx.quantize_weight(w.cuda(), layout=mx.SF_ROWMAJOR)
    assert np.array_equal(c.cpu().numpy(), ref_c)
    assert np.array_equal(s.cpu().numpy().reshape(3, 2), ref_s)


def test_gelu_kernel_vs_oracle(mx):
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(1 << 16, generator=g) * 3).to(torch.bfloat16)
    x[:8] = torch.tensor([0.0, -0.0, 1e-30, -1e-30, 60.0, -60.0, 5.5, -5.5]).to(torch.bfloat16)
    y = mx.gelu_tanh(x.cuda())
    torch.cuda.synchronize()
    got = bf16_bits(y).astype(np.int32)
    ref = oracle.gelu_tanh_bf16(bf16_bits(x)).astype(np.int32)
    # FP32 arithmetic on the GPU vs FP64 in the oracle: the BF16 results agree
    # except where the FP64 value sits within FP32 error of a rounding
    # boundary -- then they are adjacent BF16 values.
    same_sign = (got >> 15) == (ref >> 15)
    diff = np.abs(got - ref)
    assert ((diff == 0) | (same_sign & (diff == 1))).all()
    assert (diff != 0).mean() < 1e-3
