"""GPU parity of the block-scaled GEMM and the whole linear layer against the
CPU oracle: element-wise tolerance |Y - Yref| <= 2^-7 |Yref| + 1e-3 rms(Yref)
against the FP64 oracle, and bit-exact BF16 where FP32 accumulation is exact."""
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


def make_layer(M, K, N, seed, with_bias=True):
    x = synth.activations(M, K, seed)
    w = synth.weights(N, K, seed)
    b = synth.bias(N, seed) if with_bias else None
    return x, w, b


def oracle_linear(x, w, b, rows=None, cols=None):
    xq, xs = oracle.quantize_bf16(bf16_bits(x))
    wq, ws = oracle.quantize_f32(w.numpy())
    return oracle.linear(xq, xs, wq, ws, None if b is None else f16_bits(b), rows=rows, cols=cols)


def gpu_linear(mx, x, w, b):
    wq, ws = mx.quantize_weight(w.cuda())
    y = mx.linear(x.cuda(), wq, ws, None if b is None else b.cuda())
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    return bf16_values(bf16_bits(y))


@pytest.mark.parametrize("M,K,N", [
    (256, 512, 512),     # the small workload (seed 0 below)
    (1, 128, 8),         # one row, one 8-wide column chunk
    (100, 256, 256),
    (129, 384, 264),     # ragged M and N tails
    (300, 128, 520),
    (513, 640, 1024),    # several tiles in both directions
    (260, 256, 896),     # three and a half 256-wide tiles
    (131, 384, 1160),    # four 256-wide tiles and a 136-column tail
    (64, 128, 232),      # one partial tile
])
def test_linear_vs_oracle(mx, M, K, N):
    seed = 0 if (M, K, N) == (256, 512, 512) else M + N
    x, w, b = make_layer(M, K, N, seed)
    y = gpu_linear(mx, x, w, b)
    yref = oracle_linear(x, w, b)
    assert_within_tol(y, yref, f"linear {M}x{K}x{N}")
    assert np.isfinite(y).all()


# One shape per tile walk of the GEMM (equal groups of N tiles, each holding
# at most 36 MB of weight rows, when a group of that size spans at least 6 N
# tiles; else groups of 8 M tiles, or 16 when the weights exceed 48 MB), each
# with several groups, an odd group (walked in reverse) and a ragged last
# group.  Rows and columns
# are sampled in every 128 x 128 quarter of every 256 x 256 tile, so a tile
# the walk skipped or visited twice shows.
@pytest.mark.parametrize("M,K,N", [
    (300, 20480, 4864),    # N-tile groups of 7: 7 + 7 + 5 of 19 N tiles, two M tiles (ragged)
    (2600, 256, 1024),     # M-tile groups of 8: 8 + 3 of 11 M tiles, four N tiles
    (4400, 32768, 2048),   # M-tile groups of 16 (weights 67 MB): 16 + 2 of 18 M tiles
])
def test_tile_walk_covers_every_tile(mx, M, K, N):
    x, w, b = make_layer(M, K, N, M + K)
    y = gpu_linear(mx, x, w, b)
    rows = sorted({min(r, M - 1) for t in range(0, M, 128) for r in (t, t + 77, t + 127)})
    cols = sorted({min(c, N - 1) for t in range(0, N, 128) for c in (t, t + 50, t + 127)})
    yref = oracle_linear(x, w, b, rows=np.array(rows), cols=np.array(cols))
    assert_within_tol(y[np.ix_(rows, cols)], yref, f"tile walk {M}x{K}x{N}")


def test_linear_without_bias(mx):
    x, w, _ = make_layer(200, 256, 264, 11, with_bias=False)
    y = gpu_linear(mx, x, w, None)
    assert_within_tol(y, oracle_linear(x, w, None), "no bias")


def test_exact_when_accumulation_is_exact(mx):
    # small-integer codes with unit scales and small integer biases: every
    # partial sum is an integer < 2^24, so FP32 accumulation is exact in any
    # order and Y must equal BF16_RNE(Yref) bit for bit.
    rng = np.random.default_rng(5)
    M, K, N = 200, 512, 264
    xi = rng.integers(-8, 9, (M, K)).astype(np.float32)
    wi = rng.integers(-8, 9, (N, K)).astype(np.float32)
    # force amax = 256 in every block so the scale is 2^0 and codes are exact
    xi[:, ::32] = 256.0
    wi[:, ::32] = 256.0
    b = torch.tensor(rng.integers(-100, 100, N), dtype=torch.float16)
    x = torch.tensor(xi).to(torch.bfloat16)
    w = torch.tensor(wi)
    wq, ws = mx.quantize_weight(w.cuda())
    y = mx.linear(x.cuda(), wq, ws, b.cuda())
    torch.cuda.synchronize()
    yref = oracle_linear(x, w, b)
    assert np.array_equal(bf16_bits(y), oracle.bf16_rne(yref))


@pytest.mark.parametrize("N", [512, 1024])
def test_scale_placement_probe(mx, N):
    # every code is 1.0; each (row, block) and (column, block) gets its own
    # scale, so a misplaced scale byte anywhere shows up as a wrong power of
    # two in some output (N = 1024: four tiles along N)
    rng = np.random.default_rng(9)
    M, K = 256, 512
    nb = K // 32
    ex = rng.integers(-2, 3, (M, nb))
    ew = rng.integers(-2, 3, (N, nb))
    x = torch.tensor(np.repeat(2.0 ** ex, 32, axis=1), dtype=torch.float32).to(torch.bfloat16)
    w = torch.tensor(np.repeat(2.0 ** ew, 32, axis=1), dtype=torch.float32)
    # a sign pattern so that every block contributes distinguishably
    sign_x = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    x = (x.to(torch.float32) * torch.tensor(sign_x, dtype=torch.float32)).to(torch.bfloat16)
    wq, ws = mx.quantize_weight(w.cuda())
    y = mx.linear(x.cuda(), wq, ws, None)
    torch.cuda.synchronize()
    yref = oracle_linear(x, w, None)
    # products are powers of two in [2^-4, 2^4]; 512 of them sum exactly in FP32
    assert np.array_equal(bf16_bits(y), oracle.bf16_rne(yref))


def test_prequant_equals_linear(mx):
    x, w, b = make_layer(333, 256, 136, 21)
    xc, bc = x.cuda(), b.cuda()
    wq, ws = mx.quantize_weight(w.cuda())
    y1 = mx.linear(xc, wq, ws, bc)
    xq, xs = mx.quantize(xc)
    y2 = mx.gemm_prequant(xq, xs, wq, ws, bc)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_repeatable(mx):
    x, w, b = make_layer(300, 512, 512, 4)
    xc, bc = x.cuda(), b.cuda()
    wq, ws = mx.quantize_weight(w.cuda())
    y1 = mx.linear(xc, wq, ws, bc)
    y2 = mx.linear(xc, wq, ws, bc)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_empty_m_is_noop(mx):
    w = synth.weights(64, 128, 1).cuda()
    wq, ws = mx.quantize_weight(w)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    y = mx.linear(x, wq, ws, None)
    torch.cuda.synchronize()
    assert y.shape == (0, 64)


def test_single_cta_variant_in_subprocess():
    # the GEMM has a CTA-pair (default) and a single-CTA variant; the variant
    # is fixed per process, so the single-CTA one is checked in a child
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MXFP8_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(here, "test_gemm_gpu.py"), "-k", "not subprocess"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
