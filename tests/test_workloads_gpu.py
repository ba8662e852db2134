"""The block workload at small widths (all rows compared): each linear of
the block on its own, and the chained block output against the oracle's
chain."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_within_tol, bf16_bits, bf16_values, f16_bits
from mxfp8_w8a8_quantized_b200 import synth
from oracle_chain import OracleLinear, block_rows, chain_band

pytestmark = pytest.mark.gpu

HID, FFN, M, T = 512, 1024, 300, 64


def _weights(seed, blk, hidden, ffn):
    width = {synth.HIDDEN: hidden, synth.FFN: ffn}
    out = {}
    for i, (name, K, N, _) in enumerate(synth.block_linears()):
        w = synth.weights_device(width[N], width[K], seed, 10 * blk + i, "cuda").cpu().numpy()
        b = f16_bits(synth.bias_device(width[N], seed, 10 * blk + i, "cuda"))
        out[name] = OracleLinear(w, b)
    return out


def test_small_block_linears_and_chain():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    from mxfp8_w8a8_quantized_b200.workloads import Block, workspaces
    seed = 7
    x = synth.activations_device(M, HID, seed, 1000, "cuda")
    ctx = synth.activations_device(T, HID, seed, 1001, "cuda")
    blk = Block(seed, 0, "cuda", hidden=HID, ffn=FFN)
    wa, wb = workspaces(M, T, "cuda", hidden=HID, ffn=FFN)
    y, mid = blk.forward(x, ctx, wa, wb, keep=True)
    torch.cuda.synchronize()
    assert mxfp8.device_status() == 0
    lin = _weights(seed, 0, HID, FFN)
    xb = bf16_bits(x)
    # linears fed from generator inputs: single-linear tolerance, all rows
    for name, key in (("attn1.to_q", "q1"), ("attn1.to_k", "k1"), ("attn1.to_v", "v1")):
        assert_within_tol(bf16_values(bf16_bits(mid[key])), lin[name].exact(xb), name)
    cb = bf16_bits(ctx)
    for name, key in (("attn2.to_k", "k2"), ("attn2.to_v", "v2")):
        assert_within_tol(bf16_values(bf16_bits(mid[key])), lin[name].exact(cb), name)
    # chained output: within the drift band of two admissible oracle chains
    ok, stats = chain_band(bf16_values(bf16_bits(y)), bf16_values(block_rows(xb, lin)),
                           bf16_values(block_rows(xb, lin, f32acc=True)))
    assert ok, stats


def test_workspace_reuse_does_not_leak_between_blocks():
    """Two blocks in a row through the same workspaces equal the same two
    blocks through fresh workspaces."""
    from mxfp8_w8a8_quantized_b200.workloads import Block, workspaces
    seed = 8
    x = synth.activations_device(M, HID, seed, 1000, "cuda")
    ctx = synth.activations_device(T, HID, seed, 1001, "cuda")
    b0 = Block(seed, 0, "cuda", hidden=HID, ffn=FFN)
    b1 = Block(seed, 1, "cuda", hidden=HID, ffn=FFN)
    wa, wb = workspaces(M, T, "cuda", hidden=HID, ffn=FFN)
    y_shared = b1.forward(b0.forward(x, ctx, wa, wb), ctx, wa, wb)
    y_fresh = b1.forward(b0.forward(x, ctx, *workspaces(M, T, "cuda", hidden=HID, ffn=FFN)), ctx,
                         *workspaces(M, T, "cuda", hidden=HID, ffn=FFN))
    torch.cuda.synchronize()
    assert torch.equal(y_shared, y_fresh)


def test_fused_ffn_block_equals_separate_kernels():
    """The block with ffn.net.0.proj's epilogue doing GELU + quantization
    gives the same bits as GEMM -> GELU kernel -> quantizer."""
    from mxfp8_w8a8_quantized_b200.workloads import Block, workspaces
    seed = 12
    x = synth.activations_device(M, HID, seed, 1000, "cuda")
    ctx = synth.activations_device(T, HID, seed, 1001, "cuda")
    blk = Block(seed, 0, "cuda", hidden=HID, ffn=FFN)
    y_fused = blk.forward(x, ctx, *workspaces(M, T, "cuda", hidden=HID, ffn=FFN), fuse_ffn=True)
    y_sep = blk.forward(x, ctx, *workspaces(M, T, "cuda", hidden=HID, ffn=FFN), fuse_ffn=False)
    torch.cuda.synchronize()
    assert torch.equal(y_fused, y_sep)


def test_fused_projections_equal_separate_gemms():
    """q/k/v as one N = 3 hidden GEMM (and attn2's k/v as one): the same
    bits as the separate GEMMs, for every intermediate and the output."""
    from mxfp8_w8a8_quantized_b200.workloads import Block, workspaces
    seed = 13
    x = synth.activations_device(M, HID, seed, 1000, "cuda")
    ctx = synth.activations_device(T, HID, seed, 1001, "cuda")
    blk = Block(seed, 0, "cuda", hidden=HID, ffn=FFN)
    y_f, mid_f = blk.forward(x, ctx, *workspaces(M, T, "cuda", hidden=HID, ffn=FFN), keep=True, fuse_qkv=True)
    y_s, mid_s = blk.forward(x, ctx, *workspaces(M, T, "cuda", hidden=HID, ffn=FFN), keep=True, fuse_qkv=False)
    torch.cuda.synchronize()
    assert torch.equal(y_f, y_s)
    for k in ("q1", "k1", "v1", "o1", "q2", "k2", "v2", "o2"):
        assert torch.equal(mid_f[k], mid_s[k]), k


def test_step_graph_replay_equals_eager():
    """Two blocks captured as one CUDA graph: replays give the eager result,
    also after the input buffer's contents change."""
    from mxfp8_w8a8_quantized_b200.workloads import Block, StepGraph, workspaces
    seed = 14
    x = synth.activations_device(M, HID, seed, 1000, "cuda")
    ctx = synth.activations_device(T, HID, seed, 1001, "cuda")
    blocks = [Block(seed, b, "cuda", hidden=HID, ffn=FFN) for b in range(2)]
    wa, wb = workspaces(M, T, "cuda", hidden=HID, ffn=FFN)

    def step():
        y = x
        for blk in blocks:
            y = blk.forward(y, ctx, wa, wb)
        return y

    eager = step().clone()
    g = StepGraph(step)
    assert torch.equal(g.replay(), eager)
    x.copy_(synth.activations_device(M, HID, seed, 2000, "cuda"))
    eager2 = step().clone()
    assert torch.equal(g.replay(), eager2)
    assert not torch.equal(eager, eager2)
    torch.cuda.synchronize()
    from mxfp8_w8a8_quantized_b200 import mxfp8
    assert mxfp8.device_status() == 0
