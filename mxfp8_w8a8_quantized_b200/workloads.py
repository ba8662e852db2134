"""Quantized-linear workloads of the Wan2.2 A14B transformer, built from the
C-ABI layer: the FFN pair, one block's ten linears, a denoising step of 40
blocks.  Attention and norms are not part of these workloads.

Dataflow of one block (the model card, "Coverage per transformer", lists the
ten quantized linears: q/k/v/out of attn1 and attn2, ffn.net.0.proj and
ffn.net.2; the pages do not give the dataflow between them, so attention is
replaced by stand-ins that keep every shape):

    x  [M, 5120] video tokens          ctx [512, 5120] text tokens
    q1, k1, v1 = attn1.to_q/k/v(x)      one quantization of x shared by all three;
                                        one GEMM with N = 15360 (fused QKV projection)
    o1 = attn1.to_out(v1)               self-attention stand-in: identity map, output = V
    q2 = attn2.to_q(o1)
    k2, v2 = attn2.to_k/v(ctx)          one quantization of ctx shared by both;
                                        one GEMM with N = 10240
    o2 = attn2.to_out(q2)               cross-attention stand-in: output = the queries
    f  = ffn.net.0.proj(o2)             [M, 13824]
    g  = GELU_tanh(f)                   in place
    y  = ffn.net.2(g)                   [M, 5120]  -> next block's x

Every linear quantizes its BF16 input dynamically (MXFP8) before the GEMM.
The fused projections (fuse_qkv, the default) run the concatenated weights
of q/k/v (and of attn2's k/v) as one GEMM; the outputs are column slices of
one buffer and every element is computed exactly as by the separate GEMMs.
With fuse_ffn (the default), ffn.net.0.proj's epilogue applies the GELU and
quantizes for ffn.net.2 itself (mxfp8_gemm_quantize_out): f and g are never
written, and the result is bit-identical to the separate kernels.

Every kernel call goes through `timer(kind, fn, *args)` ("quant", "gemm" or
"gelu"), which the benchmark uses to time each kind; by default it just
calls fn.
"""
import torch

from . import mxfp8, synth

BLOCK_LINEARS = [name for name, _, _, _ in synth.block_linears()]


class QLinear:
    """One quantized linear: MXFP8 weight codes + tensor-core scales, F16 bias.
    `name` labels it (the model card's module name) for per-linear timing."""

    def __init__(self, wq, ws, bias, K, N, name=None):
        self.wq, self.ws, self.bias, self.K, self.N, self.name = wq, ws, bias, K, N, name

    @classmethod
    def concat(cls, parts):
        """One linear whose output rows are those of `parts` in order (the
        weights of a fused projection).  Returns (fused, views): `views` are
        linears over slices of the fused storage, in place of `parts`.  Needs
        every N % 128 == 0, so that each part's scale atoms are whole."""
        K = parts[0].K
        assert all(p.K == K and p.N % 128 == 0 for p in parts)
        fused = cls(torch.cat([p.wq for p in parts]), torch.cat([p.ws for p in parts]),
                    torch.cat([p.bias for p in parts]), K, sum(p.N for p in parts))
        views, r, sb = [], 0, 0
        for p in parts:
            nsb = mxfp8.scale_bytes(p.N, K)
            views.append(cls(fused.wq[r: r + p.N], fused.ws[sb: sb + nsb], fused.bias[r: r + p.N], K, p.N))
            r, sb = r + p.N, sb + nsb
        return fused, views

    @classmethod
    def random(cls, K, N, seed, index, device):
        w = synth.weights_device(N, K, seed, index, device)
        b = synth.bias_device(N, seed, index, device)
        wq, ws = mxfp8.quantize_weight(w)     # offline RTN weight quantization
        del w
        return cls(wq, ws, b, K, N)

    def __call__(self, xq, xs, out=None):
        return mxfp8.gemm_prequant(xq, xs, self.wq, self.ws, self.bias, out=out)

    def quantize_out(self, xq, xs, act, dest):
        """The next linear's MXFP8 input (codes, scales) from this GEMM's
        epilogue, into Workspace `dest`."""
        codes, scales = dest.views(xq.shape[0], self.N)
        return mxfp8.gemm_quantize_out(xq, xs, self.wq, self.ws, self.bias, act=act, codes=codes, scales=scales)


class Workspace:
    """Reusable activation-quantization buffers (codes + scales)."""

    def __init__(self, max_elems, max_rows, K_max, device):
        self.codes = torch.empty(max_elems, dtype=torch.uint8, device=device)
        self.scales = torch.empty(mxfp8.scale_bytes(max_rows, K_max), dtype=torch.uint8, device=device)

    def views(self, M, K):
        """(codes [M, K], tensor-core scales) views of the buffers."""
        return self.codes[: M * K].view(M, K), self.scales[: mxfp8.scale_bytes(M, K)]

    def quantize(self, x):
        codes, scales = self.views(*x.shape)
        return mxfp8.quantize(x, codes=codes, scales=scales)


class Block:
    """The ten quantized linears of one Wan block (weights random-init with
    the recipe of `synth`; linear i of block b draws stream 10 b + i)."""

    def __init__(self, seed, block_index, device, hidden=synth.HIDDEN, ffn=synth.FFN):
        self.lin = {}
        width = {synth.HIDDEN: hidden, synth.FFN: ffn}
        for i, (name, K, N, _) in enumerate(synth.block_linears()):
            self.lin[name] = QLinear.random(width[K], width[N], seed, 10 * block_index + i, device)
        L = self.lin
        self.qkv, (L["attn1.to_q"], L["attn1.to_k"], L["attn1.to_v"]) = QLinear.concat(
            [L["attn1.to_q"], L["attn1.to_k"], L["attn1.to_v"]])
        self.kv2, (L["attn2.to_k"], L["attn2.to_v"]) = QLinear.concat([L["attn2.to_k"], L["attn2.to_v"]])
        for name, lin in L.items():
            lin.name = name
        self.qkv.name, self.kv2.name = "attn1.to_qkv", "attn2.to_kv"

    def forward(self, x, ctx, ws_a, ws_b, keep=False, fuse_qkv=True, fuse_ffn=True, timer=None):
        """x [M, hidden], ctx [T, hidden] BF16.  ws_a / ws_b: two Workspaces
        (two live quantized activations at most).  Returns y, plus every
        intermediate when keep=True (g only without fuse_ffn)."""
        L = self.lin
        T = timer or _call
        H = L["attn1.to_q"].N
        xq, xs = T("quant", ws_a.quantize, x)
        if fuse_qkv:
            qkv = T("gemm", self.qkv, xq, xs)
            q1, k1, v1 = qkv[:, :H], qkv[:, H: 2 * H], qkv[:, 2 * H:]
        else:
            q1 = T("gemm", L["attn1.to_q"], xq, xs)
            k1 = T("gemm", L["attn1.to_k"], xq, xs)
            v1 = T("gemm", L["attn1.to_v"], xq, xs)
        o1 = T("gemm", L["attn1.to_out"], *T("quant", ws_b.quantize, v1))
        q2 = T("gemm", L["attn2.to_q"], *T("quant", ws_a.quantize, o1))
        cq, cs = T("quant", ws_b.quantize, ctx)
        if fuse_qkv:
            kv2 = T("gemm", self.kv2, cq, cs)
            k2, v2 = kv2[:, :H], kv2[:, H:]
        else:
            k2 = T("gemm", L["attn2.to_k"], cq, cs)
            v2 = T("gemm", L["attn2.to_v"], cq, cs)
        o2 = T("gemm", L["attn2.to_out"], *T("quant", ws_a.quantize, q2))
        oq, os_ = T("quant", ws_b.quantize, o2)
        g = None
        if fuse_ffn:
            gq, gs = T("gemm", L["ffn.net.0.proj"].quantize_out, oq, os_, mxfp8.ACT_GELU_TANH, ws_a)
        else:
            g = T("gemm", L["ffn.net.0.proj"], oq, os_)
            T("gelu", mxfp8.gelu_tanh, g, out=g)
            gq, gs = T("quant", ws_a.quantize, g)
        y = T("gemm", L["ffn.net.2"], gq, gs)
        if keep:
            return y, dict(q1=q1, k1=k1, v1=v1, o1=o1, q2=q2, k2=k2, v2=v2, o2=o2, g=g)
        return y


def _call(kind, fn, *args, **kw):
    return fn(*args, **kw)


class StepGraph:
    """A step (any function of no arguments that only launches work on the
    current stream, into buffers that stay alive) captured once as a CUDA
    graph and replayed: one launch for the whole step instead of one per
    kernel.  The first run happens outside the capture, so that every
    kernel's one-time set-up is done before capturing."""

    def __init__(self, fn):
        fn()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.out = fn()

    def replay(self):
        self.graph.replay()
        return self.out


def workspaces(M, T, device, hidden=synth.HIDDEN, ffn=synth.FFN):
    """Two workspaces big enough for every activation of a block."""
    big = max(M * ffn, M * hidden, T * hidden)
    rows = max(M, T)
    return (Workspace(big, rows, max(hidden, ffn), device), Workspace(big, rows, max(hidden, ffn), device))
