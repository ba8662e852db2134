"""GPU parity of the NVFP4 path against the CPU oracle: packed E2M1 codes
and UE4M3 scales bit-exact (both sides take the same binary32 steps), the
tensor amax and the global scale exact -- the GPU forms its global scale on
the device, the oracle forms its own from the host copy of the same tensor,
and the two must be the same binary32 value -- and the GEMM (the block-scaled
GEMM in its 4-bit mode, on CTA pairs and, in a child process, on single
CTAs) within the output tolerance."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_tol, bf16_bits, bf16_values, unswizzle
from mxfp8_w8a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    return mxfp8


def _g(mx, t):
    """(device global scale tensor, the oracle's global scale from the host
    values, host amax).  The FP32 weights are measured after rounding to
    BF16, as the weight quantizer sees them."""
    host = bf16_values(bf16_bits(t.to(torch.bfloat16)))
    amax = float(np.abs(host).max()) if host.size else 0.0
    g_ref = oracle.nvfp4_global_scale(amax)
    g_dev = mx.nvfp4_global_scale(t)
    torch.cuda.synchronize()
    assert mx.nvfp4_amax(t).item() == amax
    assert g_dev.cpu().numpy().view(np.uint32)[0] == np.float32(g_ref).view(np.uint32), (g_dev.item(), g_ref)
    return g_dev, g_ref


def _dev(g):
    """A global scale chosen by the test, as the 1-element device tensor the
    library takes."""
    return torch.tensor([g], dtype=torch.float32, device="cuda")


def test_global_scale_on_device(mx):
    """448 * 6 / amax in binary32 on the device, 1 for an all-zero tensor."""
    for t, g in ((torch.zeros(64, dtype=torch.bfloat16), 1.0),
                 (torch.full((32,), 2688.0, dtype=torch.bfloat16), 1.0),
                 (torch.full((16,), -3.0, dtype=torch.bfloat16), 896.0)):
        dg, rg = _g(mx, t.cuda())
        assert float(rg) == g and dg.item() == g


# (40000, 48): more rows than the quantizer's resident warps (32 x 148
# blocks x 8), so warps walk a second row; three blocks per row.
@pytest.mark.parametrize("M,K", [(256, 512), (1, 16), (300, 5120), (129, 13824), (1000, 1040), (64, 48),
                                 (40000, 48)])
def test_activation_quantizer_bit_exact(mx, M, K):
    x = synth.activations_device(M, K, M + K, 0, "cuda")
    g, g_ref = _g(mx, x)
    codes, scales = mx.nvfp4_quantize(x, g)
    torch.cuda.synchronize()
    rq, rs = oracle.nvfp4_quantize_bf16(bf16_bits(x), g_ref)
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
    g = float(np.float32(448.0 * 6.0 / 3.0e4))
    codes, scales = mx.nvfp4_quantize(x, _dev(g))
    torch.cuda.synchronize()
    rq, rs = oracle.nvfp4_quantize_bf16(bf16_bits(x), g)
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(unswizzle(scales.cpu().numpy(), M, K, 16), rs)
    c2, s2 = mx.nvfp4_quantize(x.contiguous(), _dev(g))
    torch.cuda.synchronize()
    assert torch.equal(codes, c2) and torch.equal(scales, s2)


@pytest.mark.parametrize("N,K", [(512, 512), (333, 13824), (8, 16)])
def test_weight_quantizer_rounds_to_bf16_first(mx, N, K):
    w = synth.weights_device(N, K, N + K, 0, "cuda")
    g, g_ref = _g(mx, w)
    wb = bf16_bits(w.to(torch.bfloat16))
    codes, scales = mx.nvfp4_quantize_weight(w, g)
    torch.cuda.synchronize()
    rq, rs = oracle.nvfp4_quantize_bf16(wb, g_ref)
    assert np.array_equal(codes.cpu().numpy(), rq)
    assert np.array_equal(unswizzle(scales.cpu().numpy(), N, K, 16), rs)


# ------------------------------------------------------------------ GEMM
# Y within |Y - Yref| <= 2^-7 |Yref| + 1e-3 rms(Yref) of the exact (FP64)
# oracle; the FP32 accumulation order is not fixed, alpha is rounded once to
# binary32.

def _nv_layer(mx, M, K, N, seed, with_bias=True):
    x = synth.activations_device(M, K, seed, 0, "cuda")
    w = synth.weights_device(N, K, seed, 0, "cuda")
    b = synth.bias_device(N, seed, 0, "cuda") if with_bias else None
    gx, gx_ref = _g(mx, x)
    gw, gw_ref = _g(mx, w)
    wq, ws = mx.nvfp4_quantize_weight(w, gw)
    return x, w, b, (gx, gx_ref), (gw, gw_ref), wq, ws


def _oracle_y(x, w, b, gx, gw, rows=None, cols=None):
    """The oracle's layer with its own (host) global scales."""
    rq, rs = oracle.nvfp4_quantize_bf16(bf16_bits(x), gx)
    oq, os_ = oracle.nvfp4_quantize_bf16(bf16_bits(w.to(torch.bfloat16)), gw)
    bb = None if b is None else b.cpu().view(torch.int16).numpy().view(np.uint16)
    return oracle.nvfp4_linear(rq, rs, gx, oq, os_, gw, bb, rows=rows, cols=cols)


@pytest.mark.parametrize("M,K,N", [(256, 512, 512), (300, 512, 384), (1, 64, 8), (129, 256, 640),
                                   (1000, 1088, 1536), (517, 13824, 264), (260, 320, 520)])
def test_gemm_within_tolerance(mx, M, K, N):
    x, w, b, (gx, gx_ref), (gw, gw_ref), wq, ws = _nv_layer(mx, M, K, N, seed=M + N)
    xq, xs = mx.nvfp4_quantize(x, gx)
    y = mx.nvfp4_gemm(xq, xs, wq, ws, gx, gw, b)
    y2 = mx.nvfp4_linear(x, gx, wq, ws, gw, b)
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    assert torch.equal(y, y2), "nvfp4_linear differs from quantize + gemm"
    yref = _oracle_y(x, w, b, gx_ref, gw_ref)
    assert_within_tol(bf16_values(bf16_bits(y)), yref, f"nvfp4 {M}x{K}x{N}")


# The tile walk is chosen on the packed row bytes (K / 2): one shape per
# walk, each with several groups, a reversed group and a ragged last group,
# sampled in every 128 x 128 quarter of every 256 x 256 tile.
@pytest.mark.parametrize("M,K,N", [
    (300, 40960, 4864),    # N-tile groups of 7: 7 + 7 + 5 of 19 N tiles
    (2600, 512, 1024),     # M-tile groups of 8: 8 + 3 of 11 M tiles
    (4400, 65536, 2048),   # M-tile groups of 16 (packed weights 67 MB): 16 + 2 of 18 M tiles
])
def test_gemm_tile_walk_covers_every_tile(mx, M, K, N):
    x, w, b, (gx, gx_ref), (gw, gw_ref), wq, ws = _nv_layer(mx, M, K, N, seed=M + N)
    xq, xs = mx.nvfp4_quantize(x, gx)
    y = mx.nvfp4_gemm(xq, xs, wq, ws, gx, gw, b)
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    rows = sorted({min(r, M - 1) for t in range(0, M, 128) for r in (t, t + 77, t + 127)})
    cols = sorted({min(c, N - 1) for t in range(0, N, 128) for c in (t, t + 50, t + 127)})
    yref = _oracle_y(x, w, b, gx_ref, gw_ref, rows=np.array(rows), cols=np.array(cols))
    got = bf16_values(bf16_bits(y))[np.ix_(rows, cols)]
    assert_within_tol(got, yref, f"nvfp4 tile walk {M}x{K}x{N}")


def test_gemm_exact_grid_values(mx):
    # every block holds a 6 and values of the E2M1 grid; with g = 1 every
    # scale is exactly 1 (6 * RN(1/6) rounds to 1 in E4M3), the codes are
    # the values themselves, and the FP32 sums are exact (multiples of 1/4
    # below 2^20), so Y is the BF16 rounding of the exact result
    M, K, N = 130, 256, 136
    grid = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    gen = torch.Generator(device="cpu").manual_seed(7)

    def make(rows):
        v = grid[torch.randint(0, 8, (rows, K), generator=gen)]
        v = v * torch.where(torch.rand((rows, K), generator=gen) < 0.5, -1.0, 1.0)
        v[:, ::16] = 6.0
        return v

    xv, wv = make(M), make(N)
    x = xv.to(torch.bfloat16).cuda()
    one = _dev(1.0)
    xq, xs = mx.nvfp4_quantize(x, one)
    wq, ws = mx.nvfp4_quantize_weight(wv.cuda(), one)
    y = mx.nvfp4_gemm(xq, xs, wq, ws, one, one, None)
    torch.cuda.synchronize()
    assert np.all(unswizzle(xs.cpu().numpy(), M, K, 16) == 0x38)
    exact = xv.double().numpy() @ wv.double().numpy().T
    assert np.array_equal(bf16_bits(y), oracle.bf16_rne(exact))


def test_gemm_q_projection_480p_full_size_sampled(mx):
    """M = 32760, K = N = 5120: codes and scales bit-exact, sampled Y."""
    M, K, N, seed = synth.TOKENS_480P, synth.HIDDEN, synth.HIDDEN, 1
    x, w, b, (gx, gx_ref), (gw, gw_ref), wq, ws = _nv_layer(mx, M, K, N, seed)
    xq, xs = mx.nvfp4_quantize(x, gx)
    y = mx.nvfp4_gemm(xq, xs, wq, ws, gx, gw, b)
    torch.cuda.synchronize()
    assert mx.device_status() == 0
    rq, rs = oracle.nvfp4_quantize_bf16(bf16_bits(x), gx_ref)
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(unswizzle(xs.cpu().numpy(), M, K, 16), rs)
    oq, os_ = oracle.nvfp4_quantize_bf16(bf16_bits(w.to(torch.bfloat16)), gw_ref)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, M - 129, M - 1], np.arange(M - 40, M),
                                     rng.choice(M, 150, replace=False)]))
    cols = np.unique(np.concatenate([[0, 8, 255, 256, N - 1], rng.choice(N, 120, replace=False)]))
    bb = b.cpu().view(torch.int16).numpy().view(np.uint16)
    yref = oracle.nvfp4_linear(rq, rs, gx_ref, oq, os_, gw_ref, bb, rows=rows, cols=cols)
    got = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
    assert_within_tol(bf16_values(bf16_bits(got)), yref, "nvfp4 Q projection")


def test_gemm_argument_errors(mx):
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device="cuda")
    one = _dev(1.0)
    xq, xs = mx.nvfp4_quantize(x, one)
    w = torch.zeros((8, 96), dtype=torch.float32, device="cuda")
    wq, ws = mx.nvfp4_quantize_weight(w, one)
    with pytest.raises(mx.MXFP8Error):          # K = 96 is not a multiple of 64
        mx.nvfp4_gemm(xq, xs, wq, ws, one, one)
    with pytest.raises(ValueError):             # a global scale is a 1-element FP32 CUDA tensor
        mx.nvfp4_gemm(xq, xs, wq, ws, 1.0, one)
    with pytest.raises(ValueError):
        mx.nvfp4_quantize(x, torch.ones(2, device="cuda"))


def test_gemm_single_cta_variant_in_subprocess():
    # the GEMM has a CTA-pair (default) and a single-CTA variant, fixed per
    # process; the NVFP4 GEMM checks run again in a child on single CTAs
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, MXFP8_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(here, "test_nvfp4_gpu.py"), "-k", "gemm and not subprocess"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
