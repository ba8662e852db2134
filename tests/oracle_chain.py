"""Chains of linears computed by the CPU oracle on a few rows (test helper).

Each linear is quantize -> FP64 linear -> BF16 RNE, GELU is FP64 -> BF16,
exactly as the layer is defined; only the selected token rows are computed,
which is exact because every step acts on one token row at a time.  Weights
are quantized by the oracle itself from the same generator output the GPU
path gets.  Nothing here reads a GPU result.
"""
import numpy as np

import oracle


class OracleLinear:
    def __init__(self, w_f32: np.ndarray, b_bits: np.ndarray):
        self.wq, self.ws = oracle.quantize_f32(w_f32)
        self.b = b_bits

    def exact(self, x_bits: np.ndarray, f32acc: bool = False) -> np.ndarray:
        """Output of the layer for BF16 input rows before the BF16 rounding:
        exact (FP64), or FP32-accumulated in increasing k."""
        xq, xs = oracle.quantize_bf16(x_bits)
        f = oracle.linear_f32acc if f32acc else oracle.linear
        return f(xq, xs, self.wq, self.ws, self.b)

    def __call__(self, x_bits: np.ndarray, f32acc: bool = False) -> np.ndarray:
        return oracle.bf16_rne(self.exact(x_bits, f32acc))


def block_rows(x_bits, lin, f32acc=False):
    """The block's chain (see mxfp8_w8a8_quantized_b200.workloads) for the
    given video-token rows; `lin` maps linear name -> OracleLinear.  The text
    branch (attn2.to_k / to_v) does not feed y and is not computed here."""
    v1 = lin["attn1.to_v"](x_bits, f32acc)
    o1 = lin["attn1.to_out"](v1, f32acc)
    q2 = lin["attn2.to_q"](o1, f32acc)
    o2 = lin["attn2.to_out"](q2, f32acc)
    f = lin["ffn.net.0.proj"](o2, f32acc)
    g = oracle.gelu_tanh_bf16(f)
    return lin["ffn.net.2"](g, f32acc)


def rel_row_error(y: np.ndarray, yref: np.ndarray) -> np.ndarray:
    """Per-row ||y - yref|| / ||yref||."""
    num = np.sqrt(((y - yref) ** 2).sum(axis=1))
    den = np.sqrt((yref ** 2).sum(axis=1))
    return num / np.maximum(den, 1e-300)


# Default band (the reduced-width block of tests/test_workloads_gpu.py): the
# GPU chain's drift from the exact chain within twice the drift between two
# admissible oracle evaluations (FP64 vs FP32 in k order), plus fixed slacks.
CHAIN_FACTOR = 2.0
CHAIN_MEAN_SLACK = 2e-3
CHAIN_MAX_SLACK = 3e-2


def chain_band(got, ref64, ref32, factor=CHAIN_FACTOR, mean_slack=CHAIN_MEAN_SLACK, max_slack=CHAIN_MAX_SLACK):
    """(ok, stats): the GPU chain's per-row relative drift from the exact
    chain against the reference drift of the FP32-in-order oracle chain:
    mean D_gpu <= factor mean D_ref + mean_slack, and the same for the max."""
    d_gpu = rel_row_error(got, ref64)
    d_ref = rel_row_error(ref32, ref64)
    stats = dict(rows=len(got), gpu_mean=float(d_gpu.mean()), gpu_max=float(d_gpu.max()),
                 ref_mean=float(d_ref.mean()), ref_max=float(d_ref.max()))
    ok = (np.isfinite(got).all()
          and d_gpu.mean() <= factor * d_ref.mean() + mean_slack
          and d_gpu.max() <= factor * d_ref.max() + max_slack)
    return ok, stats
