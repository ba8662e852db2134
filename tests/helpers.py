"""Shared test helpers: conversions, the output tolerance, and the tensor-core
scale layout written out from its definition (include/mxfp8.h) so that tests
can compare the GPU's scales with the oracle's row-major ones."""
import numpy as np
import torch


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def tc_index(rows: int, K: int, block: int = 32):
    """For every (r, b) of a [rows, K/block] scale matrix, its byte offset in
    the tensor-core layout: 512-byte atoms of 128 rows x 4 blocks, atom (i, j)
    at (i * ceil(K/(4 block)) + j) * 512, byte (r, b) inside at
    (r%32)*16 + (r//32 % 4)*4 + b%4."""
    nb = K // block
    kg = (nb + 3) // 4
    r = np.arange(rows)[:, None]
    b = np.arange(nb)[None, :]
    return ((r // 128) * kg + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)


def tc_bytes(rows: int, K: int) -> int:
    return ((rows + 127) // 128) * ((K + 127) // 128) * 512


def unswizzle(sc: np.ndarray, rows: int, K: int, block: int = 32) -> np.ndarray:
    return sc[tc_index(rows, K, block)]


def tol_violations(y: np.ndarray, yref: np.ndarray):
    """|y - yref| <= 2^-7 |yref| + 1e-3 rms(yref); returns (bad mask, bound)."""
    rms = float(np.sqrt(np.mean(yref ** 2))) if yref.size else 0.0
    bound = 2.0 ** -7 * np.abs(yref) + 1e-3 * rms
    return np.abs(y - yref) > bound, bound


def assert_within_tol(y: np.ndarray, yref: np.ndarray, what=""):
    bad, bound = tol_violations(y, yref)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        det = [(tuple(i), float(y[tuple(i)]), float(yref[tuple(i)]), float(bound[tuple(i)])) for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance, e.g. {det}")


def mx_values(codes: np.ndarray, scales_rowmajor: np.ndarray, block: int = 32) -> np.ndarray:
    """Dequantized MXFP8 values (FP64) of E4M3 codes [rows, K] with E8M0
    scales [rows, K/block], decoded with torch's float8_e4m3fn."""
    c = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    e = scales_rowmajor.astype(np.float64) - 127.0
    return c * np.repeat(np.exp2(e), block, axis=1)
