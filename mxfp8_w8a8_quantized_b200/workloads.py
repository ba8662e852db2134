"""Quantized-linear workloads of the Wan2.2 A14B transformer, built from the
C-ABI layer: the FFN pair, one block's ten linears, a denoising step of 40
blocks.  Attention and norms are not part of these workloads.

Dataflow of one block (the model card, "Coverage per transformer", lists the
ten quantized linears: q/k/v/out of attn1 and attn2, ffn.net.0.proj and
ffn.net.2; the pages do not give the dataflow between them, so attention is
replaced by stand-ins that keep every shape):

    x  [M, 5120] video tokens          ctx [512, 5120] text tokens
    q1, k1, v1 = attn1.to_q/k/v(x)      one quantization of x shared by all three
    o1 = attn1.to_out(v1)               self-attention stand-in: identity map, output = V
    q2 = attn2.to_q(o1)
    k2, v2 = attn2.to_k/v(ctx)          one quantization of ctx shared by both
    o2 = attn2.to_out(q2)               cross-attention stand-in: output = the queries
    f  = ffn.net.0.proj(o2)             [M, 13824]
    g  = GELU_tanh(f)                   in place
    y  = ffn.net.2(g)                   [M, 5120]  -> next block's x

Every linear quantizes its BF16 input dynamically (MXFP8) before the GEMM.
"""
import torch

from . import mxfp8, synth

BLOCK_LINEARS = [name for name, _, _, _ in synth.block_linears()]


class QLinear:
    """One quantized linear: MXFP8 weight codes + tensor-core scales, F16 bias."""

    def __init__(self, wq, ws, bias, K, N):
        self.wq, self.ws, self.bias, self.K, self.N = wq, ws, bias, K, N

    @classmethod
    def random(cls, K, N, seed, index, device):
        w = synth.weights_device(N, K, seed, index, device)
        b = synth.bias_device(N, seed, index, device)
        wq, ws = mxfp8.quantize_weight(w)     # offline RTN weight quantization
        del w
        return cls(wq, ws, b, K, N)

    def __call__(self, xq, xs, out=None):
        return mxfp8.gemm_prequant(xq, xs, self.wq, self.ws, self.bias, out=out)


class Workspace:
    """Reusable activation-quantization buffers (codes + scales)."""

    def __init__(self, max_elems, max_rows, K_max, device):
        self.codes = torch.empty(max_elems, dtype=torch.uint8, device=device)
        self.scales = torch.empty(mxfp8.scale_bytes(max_rows, K_max), dtype=torch.uint8, device=device)

    def quantize(self, x):
        M, K = x.shape
        codes = self.codes[: M * K].view(M, K)
        scales = self.scales[: mxfp8.scale_bytes(M, K)]
        return mxfp8.quantize(x, codes=codes, scales=scales)


class Block:
    """The ten quantized linears of one Wan block (weights random-init with
    the recipe of `synth`; linear i of block b draws stream 10 b + i)."""

    def __init__(self, seed, block_index, device, hidden=synth.HIDDEN, ffn=synth.FFN):
        self.lin = {}
        width = {synth.HIDDEN: hidden, synth.FFN: ffn}
        for i, (name, K, N, _) in enumerate(synth.block_linears()):
            self.lin[name] = QLinear.random(width[K], width[N], seed, 10 * block_index + i, device)

    def forward(self, x, ctx, ws_a, ws_b, keep=False):
        """x [M, hidden], ctx [T, hidden] BF16.  ws_a / ws_b: two Workspaces
        (two live quantized activations at most).  Returns y, plus every
        intermediate when keep=True."""
        L = self.lin
        xq, xs = ws_a.quantize(x)
        q1 = L["attn1.to_q"](xq, xs)
        k1 = L["attn1.to_k"](xq, xs)
        v1 = L["attn1.to_v"](xq, xs)
        o1 = L["attn1.to_out"](*ws_b.quantize(v1))
        q2 = L["attn2.to_q"](*ws_a.quantize(o1))
        cq, cs = ws_b.quantize(ctx)
        k2 = L["attn2.to_k"](cq, cs)
        v2 = L["attn2.to_v"](cq, cs)
        o2 = L["attn2.to_out"](*ws_a.quantize(q2))
        f = L["ffn.net.0.proj"](*ws_b.quantize(o2))
        mxfp8.gelu_tanh(f, out=f)
        y = L["ffn.net.2"](*ws_a.quantize(f))
        if keep:
            return y, dict(q1=q1, k1=k1, v1=v1, o1=o1, q2=q2, k2=k2, v2=v2, o2=o2, g=f)
        return y


def workspaces(M, T, device, hidden=synth.HIDDEN, ffn=synth.FFN):
    """Two workspaces big enough for every activation of a block."""
    big = max(M * ffn, M * hidden, T * hidden)
    rows = max(M, T)
    return (Workspace(big, rows, max(hidden, ffn), device), Workspace(big, rows, max(hidden, ffn), device))
