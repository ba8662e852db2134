"""CPU oracle for the MXFP8 W8A8 linear layer (numpy front end).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` are the only callers.  The product path
(``mxfp8_w8a8_quantized_b200``) never imports this package, and this package
never imports the product.  The arithmetic lives in ``mxfp8_oracle.c``; this
file only marshals numpy arrays.

What each function computes, and the passage it follows, is stated in the
header of ``mxfp8_oracle.c`` (model card "Wan2.2-I2V-A14B-Lightning . MXFP8
(AutoRound OptRTN)", sections "Quantization Details" and "Coverage per
transformer").  Every function here has a pin in tests/test_oracle_*.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        # ORACLE_LIB lets the mutation test load a deliberately broken copy
        path = os.environ.get("ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_decode.restype = ctypes.c_double
        L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
        L.orc_bf16_decode.restype = ctypes.c_double
        L.orc_f16_decode.argtypes = [ctypes.c_uint16]
        L.orc_f16_decode.restype = ctypes.c_double
        L.orc_bf16_rne.argtypes = [ctypes.c_double]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_gelu_tanh.argtypes = [ctypes.c_double]
        L.orc_gelu_tanh.restype = ctypes.c_double
        L.orc_quantize_block_f64.argtypes = [P, ctypes.c_int, P, P]
        L.orc_quantize_bf16.argtypes = [P, I64, I64, I64, P, P]
        L.orc_quantize_f32.argtypes = [P, I64, I64, P, P]
        L.orc_dequantize.argtypes = [P, P, I64, I64, P]
        L.orc_linear.argtypes = [P, P, I64, I64, P, P, I64, P, P, I64, P, I64, P]
        L.orc_linear_f32acc.argtypes = [P, P, I64, I64, P, P, I64, P, P, I64, P, I64, P]
        L.orc_bf16_rne_array.argtypes = [P, I64, P]
        L.orc_gelu_tanh_bf16.argtypes = [P, I64, P]
        L.orc_quantize_rowwise_bf16.argtypes = [P, I64, I64, I64, P, P]
        L.orc_quantize_rowwise_f32.argtypes = [P, I64, I64, P, P]
        L.orc_linear_rowwise.argtypes = [P, P, I64, I64, P, P, I64, P, P, I64, P, I64, P]
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_encode.argtypes = [ctypes.c_double]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_nvfp4_quantize_bf16.argtypes = [P, I64, I64, I64, ctypes.c_float, P, P]
        L.orc_nvfp4_dequantize.argtypes = [P, P, I64, I64, ctypes.c_float, P]
        L.orc_nvfp4_linear.argtypes = [P, P, ctypes.c_float, I64, I64, P, P, ctypes.c_float, I64, P, P, I64, P,
                                       I64, P]
        L.orc_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars
def e4m3_decode(codes):
    """E4M3 code(s) -> float64 value(s)."""
    c = np.asarray(codes, dtype=np.uint8)
    f = np.vectorize(lambda v: lib().orc_e4m3_decode(int(v)), otypes=[np.float64])
    return f(c)


def e4m3_encode(values):
    """Real value(s) -> nearest E4M3 code(s), ties to even, saturating at 448."""
    v = np.asarray(values, dtype=np.float64)
    f = np.vectorize(lambda x: lib().orc_e4m3_encode(float(x)), otypes=[np.uint8])
    return f(v)


def e8m0_decode(b):
    v = np.asarray(b, dtype=np.uint8)
    f = np.vectorize(lambda x: lib().orc_e8m0_decode(int(x)), otypes=[np.float64])
    return f(v)


def f16_decode(bits):
    v = np.asarray(bits, dtype=np.uint16)
    f = np.vectorize(lambda x: lib().orc_f16_decode(int(x)), otypes=[np.float64])
    return f(v)


def bf16_decode(bits):
    v = np.asarray(bits, dtype=np.uint16)
    f = np.vectorize(lambda x: lib().orc_bf16_decode(int(x)), otypes=[np.float64])
    return f(v)


def bf16_rne(values):
    """float64 array -> BF16 bit patterns (uint16), round to nearest even."""
    v = _c(values, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_bf16_rne_array(_ptr(v), v.size, _ptr(out))
    return out


def gelu_tanh(x):
    f = np.vectorize(lambda t: lib().orc_gelu_tanh(float(t)), otypes=[np.float64])
    return f(np.asarray(x, dtype=np.float64))


def gelu_tanh_bf16(x_bits):
    """BF16 bits in -> GELU(tanh) in FP64 -> BF16 bits out."""
    x = _c(x_bits, np.uint16)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_gelu_tanh_bf16(_ptr(x), x.size, _ptr(out))
    return out


# ---------------------------------------------------------------- quantizer
def quantize_block(values):
    """One block of float64 values -> (codes uint8[n], scale byte)."""
    x = _c(values, np.float64)
    codes = np.empty(x.size, dtype=np.uint8)
    sc = np.zeros(1, dtype=np.uint8)
    lib().orc_quantize_block_f64(_ptr(x), x.size, _ptr(codes), _ptr(sc))
    return codes, int(sc[0])


def quantize_bf16(x_bits):
    """BF16 bits [R, K] -> (codes uint8 [R, K], scales uint8 [R, K/32])."""
    x = _c(x_bits, np.uint16)
    R, K = x.shape
    assert K % 32 == 0
    codes = np.empty((R, K), dtype=np.uint8)
    scales = np.empty((R, K // 32), dtype=np.uint8)
    lib().orc_quantize_bf16(_ptr(x), R, K, K, _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_f32(w):
    """FP32 [R, K] -> (codes uint8 [R, K], scales uint8 [R, K/32])."""
    x = _c(w, np.float32)
    R, K = x.shape
    assert K % 32 == 0
    codes = np.empty((R, K), dtype=np.uint8)
    scales = np.empty((R, K // 32), dtype=np.uint8)
    lib().orc_quantize_f32(_ptr(x), R, K, _ptr(codes), _ptr(scales))
    return codes, scales


def dequantize(codes, scales):
    c = _c(codes, np.uint8)
    s = _c(scales, np.uint8)
    R, K = c.shape
    out = np.empty((R, K), dtype=np.float64)
    lib().orc_dequantize(_ptr(c), _ptr(s), R, K, _ptr(out))
    return out


# ---------------------------------------------------------------- linear
def linear(xq, xs, wq, ws, bias_bits=None, rows=None, cols=None):
    """Y = Xhat What^T + bias in FP64 for the selected rows / columns.

    xq [M, K] / xs [M, K/32]; wq [N, K] / ws [N, K/32]; bias F16 bits [N].
    """
    xq = _c(xq, np.uint8)
    xs = _c(xs, np.uint8)
    wq = _c(wq, np.uint8)
    ws = _c(ws, np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K and xs.shape == (M, K // 32) and ws.shape == (N, K // 32)
    r = None if rows is None else _c(rows, np.int64)
    c = None if cols is None else _c(cols, np.int64)
    nr = M if r is None else r.size
    nc = N if c is None else c.size
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    Y = np.empty((nr, nc), dtype=np.float64)
    lib().orc_linear(_ptr(xq), _ptr(xs), M, K, _ptr(wq), _ptr(ws), N, _ptr(b),
                     _ptr(r), nr, _ptr(c), nc, _ptr(Y))
    return Y


def linear_f32acc(xq, xs, wq, ws, bias_bits=None, rows=None, cols=None):
    """As `linear`, but accumulated in FP32 in increasing k (one admissible
    FP32 evaluation order); returns the FP32 results as float64."""
    xq = _c(xq, np.uint8)
    xs = _c(xs, np.uint8)
    wq = _c(wq, np.uint8)
    ws = _c(ws, np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    r = None if rows is None else _c(rows, np.int64)
    c = None if cols is None else _c(cols, np.int64)
    nr = M if r is None else r.size
    nc = N if c is None else c.size
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    Y = np.empty((nr, nc), dtype=np.float64)
    lib().orc_linear_f32acc(_ptr(xq), _ptr(xs), M, K, _ptr(wq), _ptr(ws), N, _ptr(b),
                            _ptr(r), nr, _ptr(c), nc, _ptr(Y))
    return Y


def num_threads():
    return int(lib().orc_num_threads())


# ------------------------------------------------------ per-channel FP8
def quantize_rowwise_bf16(x_bits):
    """BF16 bits [M, K] -> (E4M3 codes [M, K], FP32 scales [M]); one scale
    amax / 448 per row, codes E4M3(x / s) (binary32 divisions)."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    lib().orc_quantize_rowwise_bf16(_ptr(x), M, K, K, _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_rowwise_f32(w):
    """FP32 [N, K] -> (E4M3 codes [N, K], FP32 scales [N]), one per output channel."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty(N, dtype=np.float32)
    lib().orc_quantize_rowwise_f32(_ptr(w), N, K, _ptr(codes), _ptr(scales))
    return codes, scales


def linear_rowwise(xq, sx, wq, sw, bias_bits=None, rows=None, cols=None):
    """Exact per-channel FP8 linear for the selected rows / cols (FP64)."""
    xq = _c(xq, np.uint8)
    wq = _c(wq, np.uint8)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    r = None if rows is None else _c(rows, np.int64)
    c = None if cols is None else _c(cols, np.int64)
    nr = M if r is None else len(r)
    nc = N if c is None else len(c)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((nr, nc), dtype=np.float64)
    lib().orc_linear_rowwise(_ptr(xq), _ptr(sx), M, K, _ptr(wq), _ptr(sw), N, _ptr(b), _ptr(r), nr, _ptr(c), nc,
                             _ptr(y))
    return y


# ------------------------------------------------------------------ NVFP4
def e2m1_decode(codes):
    """E2M1 code(s) (0..15) -> float64 value(s)."""
    c = np.asarray(codes, dtype=np.uint8)
    f = np.vectorize(lambda v: lib().orc_e2m1_decode(int(v)), otypes=[np.float64])
    return f(c)


def e2m1_encode(values):
    """Real value(s) -> nearest E2M1 code(s), ties to even, saturating at 6."""
    v = np.asarray(values, dtype=np.float64)
    f = np.vectorize(lambda x: lib().orc_e2m1_encode(float(x)), otypes=[np.uint8])
    return f(v)


def nvfp4_quantize_bf16(x_bits, g):
    """BF16 bits [M, K] and global scale g -> (packed E2M1 codes [M, K/2],
    UE4M3 scales [M, K/16])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K // 2), dtype=np.uint8)
    scales = np.empty((M, K // 16), dtype=np.uint8)
    lib().orc_nvfp4_quantize_bf16(_ptr(x), M, K, K, float(np.float32(g)), _ptr(codes), _ptr(scales))
    return codes, scales


def nvfp4_dequantize(codes, scales, g):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    M = codes.shape[0]
    K = codes.shape[1] * 2
    out = np.empty((M, K), dtype=np.float64)
    lib().orc_nvfp4_dequantize(_ptr(codes), _ptr(scales), M, K, float(np.float32(g)), _ptr(out))
    return out


def nvfp4_linear(xq, xs, gx, wq, ws, gw, bias_bits=None, rows=None, cols=None):
    """Exact NVFP4 linear for the selected rows / cols (FP64)."""
    xq = _c(xq, np.uint8)
    xs = _c(xs, np.uint8)
    wq = _c(wq, np.uint8)
    ws = _c(ws, np.uint8)
    M = xq.shape[0]
    K = xq.shape[1] * 2
    N = wq.shape[0]
    r = None if rows is None else _c(rows, np.int64)
    c = None if cols is None else _c(cols, np.int64)
    nr = M if r is None else len(r)
    nc = N if c is None else len(c)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((nr, nc), dtype=np.float64)
    lib().orc_nvfp4_linear(_ptr(xq), _ptr(xs), float(np.float32(gx)), M, K, _ptr(wq), _ptr(ws),
                           float(np.float32(gw)), N, _ptr(b), _ptr(r), nr, _ptr(c), nc, _ptr(y))
    return y


def nvfp4_global_scale(amax):
    """The per-tensor global scale 448 * 6 / amax (binary32 division): the
    largest block then gets the largest UE4M3 scale.  When amax is 0 or not
    finite, or the quotient overflows, no finite scale maps the tensor onto
    the format's range and the scale is 1 (reading: the page gives the field,
    not its value for an all-zero tensor)."""
    a = np.float32(amax)
    if not (a > 0 and np.isfinite(a)):
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        q = np.float32(np.float32(448.0 * 6.0) / a)
    return q if np.isfinite(q) else np.float32(1.0)
