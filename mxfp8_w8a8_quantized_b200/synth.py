"""Seeded synthetic inputs for the MXFP8 W8A8 linear layer.

This module only draws random numbers; it holds none of the method's
arithmetic.  Tests give the same tensors to the CUDA path and to the CPU
oracle, and ``bench.py`` times the CUDA path on them.

Workload recipe (the pages ship no activations or weights, so these stand in
for them):

* X, BF16 [M, K]: N(0, 1), with round(0.01 K) distinct input channels
  (columns, chosen with the same seed) multiplied by 20 -- outlier channels.
* W, FP32 [N, K] (out x in, K contiguous): N(0, std = 1/sqrt(K)); quantized
  offline to MXFP8 by round-to-nearest.
* bias, F16 [N]: N(0, std = 0.01).  The model card ("Coverage per
  transformer") keeps the biases of the 400 quantized linears in F16.

Token counts follow Wan2.2's latent grid for 81 frames (21 latent frames)
with a 16x spatial reduction: 480x832 -> 21*30*52 = 32760 tokens, 832x1104
(the model card's example resolution) -> 21*69*52 = 75348 tokens; the text
context is 512 tokens.  Widths are the A14B hidden size 5120 and FFN size
13824; each block has 10 quantized linears (model card, "Coverage per
transformer": q/k/v/out of attn1 and attn2, ffn.net.0.proj, ffn.net.2).
"""
import torch

HIDDEN = 5120
FFN = 13824
TEXT_TOKENS = 512
TOKENS_480P = 32760    # 21 x 30 x 52
TOKENS_832x1104 = 75348  # 21 x 69 x 52
BLOCKS = 40

# stream tags: every tensor of a workload has its own generator stream
_TAG_X, _TAG_W, _TAG_B, _TAG_CH = 1, 2, 3, 4


def _gen(seed: int, tag: int, index: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * 1_000_003 + tag * 10_007 + index) & 0x7FFF_FFFF_FFFF)
    return g


def outlier_channels(K: int, seed: int, index: int = 0, frac: float = 0.01) -> torch.Tensor:
    """round(frac*K) distinct channel indices, sorted."""
    n = int(round(frac * K))
    g = _gen(seed, _TAG_CH, index)
    return torch.sort(torch.randperm(K, generator=g)[:n]).values


def activations(M: int, K: int, seed: int, index: int = 0, outliers: bool = True,
                gain: float = 20.0) -> torch.Tensor:
    """BF16 [M, K] on the CPU: N(0,1) with 1% of channels scaled by `gain`."""
    g = _gen(seed, _TAG_X, index)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if outliers:
        ch = outlier_channels(K, seed, index)
        x[:, ch] *= gain
    return x.to(torch.bfloat16)


def weights(N: int, K: int, seed: int, index: int = 0) -> torch.Tensor:
    """FP32 [N, K] on the CPU: N(0, 1/sqrt(K))."""
    g = _gen(seed, _TAG_W, index)
    return torch.randn(N, K, generator=g, dtype=torch.float32) * (1.0 / K ** 0.5)


def bias(N: int, seed: int, index: int = 0) -> torch.Tensor:
    """F16 [N] on the CPU: N(0, 0.01)."""
    g = _gen(seed, _TAG_B, index)
    return (torch.randn(N, generator=g, dtype=torch.float32) * 0.01).to(torch.float16)


def weights_device(N: int, K: int, seed: int, index: int, device) -> torch.Tensor:
    """FP32 [N, K] drawn on `device` (for workloads too large to draw on the
    host); same distribution as `weights`, different stream."""
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + _TAG_W * 10_007 + index) & 0x7FFF_FFFF_FFFF)
    return torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * (1.0 / K ** 0.5)


def bias_device(N: int, seed: int, index: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + _TAG_B * 10_007 + index) & 0x7FFF_FFFF_FFFF)
    return (torch.randn(N, generator=g, dtype=torch.float32, device=device) * 0.01).to(torch.float16)


def activations_device(M: int, K: int, seed: int, index: int, device, outliers: bool = True,
                       gain: float = 20.0) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + _TAG_X * 10_007 + index) & 0x7FFF_FFFF_FFFF)
    x = torch.randn(M, K, generator=g, dtype=torch.float32, device=device)
    if outliers:
        ch = outlier_channels(K, seed, index).to(device)
        x[:, ch] *= gain
    return x.to(torch.bfloat16)


# The five workloads: (name, description).  Shapes are Y[M,N] = X[M,K] W[N,K]^T.
WORKLOADS = {
    "c0_small": dict(seed=0, M=256, K=512, N=512),
    "c1_q_proj_480p": dict(seed=1, M=TOKENS_480P, K=HIDDEN, N=HIDDEN),
    "c2_ffn_pair_832x1104": dict(seed=2, M=TOKENS_832x1104, K=HIDDEN, N=FFN),
    "c3_block_832x1104": dict(seed=3, M=TOKENS_832x1104, K=HIDDEN, N=HIDDEN),
    "c4_step_832x1104": dict(seed=4, M=TOKENS_832x1104, K=HIDDEN, N=HIDDEN, blocks=BLOCKS),
}


def block_linears():
    """The 10 quantized linears of one Wan block as (name, K, N, token kind).

    Token kind "video" runs on the video tokens, "text" on the 512 text tokens.
    """
    return [
        ("attn1.to_q", HIDDEN, HIDDEN, "video"),
        ("attn1.to_k", HIDDEN, HIDDEN, "video"),
        ("attn1.to_v", HIDDEN, HIDDEN, "video"),
        ("attn1.to_out", HIDDEN, HIDDEN, "video"),
        ("attn2.to_q", HIDDEN, HIDDEN, "video"),
        ("attn2.to_k", HIDDEN, HIDDEN, "text"),
        ("attn2.to_v", HIDDEN, HIDDEN, "text"),
        ("attn2.to_out", HIDDEN, HIDDEN, "video"),
        ("ffn.net.0.proj", HIDDEN, FFN, "video"),
        ("ffn.net.2", FFN, HIDDEN, "video"),
    ]
