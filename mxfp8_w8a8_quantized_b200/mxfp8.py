"""Thin ctypes binding over libmxfp8.so (C-ABI in include/mxfp8.h).

Argument marshalling only: tensors are passed as device pointers together
with the current CUDA stream, outputs are allocated with PyTorch.  Every step
of the layer runs in the library's kernels; there is no CPU or library
fallback, and importing this module raises if the library is missing.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxfp8.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m mxfp8_w8a8_quantized_b200.build` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

_lib.mxfp8_status_str.argtypes = [ctypes.c_int]
_lib.mxfp8_status_str.restype = ctypes.c_char_p
_lib.mxfp8_scale_bytes.argtypes = [_I64, _I64, ctypes.c_int]
_lib.mxfp8_scale_bytes.restype = _SZ
_lib.mxfp8_quantize.argtypes = [_P, _I64, _I64, _I64, _P, _P, ctypes.c_int, _P]
_lib.mxfp8_quantize.restype = ctypes.c_int
_lib.mxfp8_quantize_weight_f32.argtypes = [_P, _I64, _I64, _P, _P, ctypes.c_int, _P]
_lib.mxfp8_quantize_weight_f32.restype = ctypes.c_int
_lib.mxfp8_linear_workspace_bytes.argtypes = [_I64, _I64]
_lib.mxfp8_linear_workspace_bytes.restype = _SZ
_lib.mxfp8_linear.argtypes = [_P, _I64, _I64, _P, _P, _I64, _P, _P, _P, _SZ, _P]
_lib.mxfp8_linear.restype = ctypes.c_int
_lib.mxfp8_gemm_prequant.argtypes = [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P, _P]
_lib.mxfp8_gemm_prequant.restype = ctypes.c_int
_lib.mxfp8_gelu_tanh_bf16.argtypes = [_P, _P, _I64, _P]
_lib.mxfp8_gelu_tanh_bf16.restype = ctypes.c_int
_lib.mxfp8_linear_noalloc.argtypes = [_P, _I64, _I64, _P, _P, _I64, _P, _P, _P]
_lib.mxfp8_linear_noalloc.restype = ctypes.c_int
_lib.mxfp8_gemm_quantize_out.argtypes = [_P, _P, _I64, _I64, _P, _P, _I64, _P, ctypes.c_int, _P, _P, _P]
_lib.mxfp8_gemm_quantize_out.restype = ctypes.c_int
_lib.fp8rw_quantize_bf16.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P]
_lib.fp8rw_quantize_bf16.restype = ctypes.c_int
_lib.fp8rw_quantize_weight_f32.argtypes = [_P, _I64, _I64, _P, _P, _P]
_lib.fp8rw_quantize_weight_f32.restype = ctypes.c_int
_lib.fp8rw_gemm.argtypes = [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P, _P]
_lib.fp8rw_gemm.restype = ctypes.c_int
_lib.fp8rw_linear_workspace_bytes.argtypes = [_I64, _I64]
_lib.fp8rw_linear_workspace_bytes.restype = _SZ
_lib.fp8rw_linear.argtypes = [_P, _I64, _I64, _P, _P, _I64, _P, _P, _P, _SZ, _P]
_lib.fp8rw_linear.restype = ctypes.c_int
_lib.nvfp4_scale_bytes.argtypes = [_I64, _I64]
_lib.nvfp4_scale_bytes.restype = _SZ
_lib.nvfp4_amax_bf16.argtypes = [_P, _I64, _P, _P]
_lib.nvfp4_amax_bf16.restype = ctypes.c_int
_lib.nvfp4_amax_f32.argtypes = [_P, _I64, _P, _P]
_lib.nvfp4_amax_f32.restype = ctypes.c_int
_lib.nvfp4_global_scale_from_amax.argtypes = [_P, _P, _P]
_lib.nvfp4_global_scale_from_amax.restype = ctypes.c_int
_lib.nvfp4_quantize_bf16.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _P]
_lib.nvfp4_quantize_bf16.restype = ctypes.c_int
_lib.nvfp4_quantize_weight_f32.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]
_lib.nvfp4_quantize_weight_f32.restype = ctypes.c_int
_lib.nvfp4_gemm.argtypes = [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P, _P, _P, _P]
_lib.nvfp4_gemm.restype = ctypes.c_int
_lib.nvfp4_linear_workspace_bytes.argtypes = [_I64, _I64]
_lib.nvfp4_linear_workspace_bytes.restype = _SZ
_lib.nvfp4_linear.argtypes = [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _P, _SZ, _P]
_lib.nvfp4_linear.restype = ctypes.c_int
_lib.mxfp8_selftest_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_uint64, _P]
_lib.mxfp8_selftest_wait_timeout.restype = ctypes.c_int
_lib.mxfp8_device_status.argtypes = [_P]
_lib.mxfp8_device_status.restype = ctypes.c_int

SF_ROWMAJOR = 0
SF_TCGEN05 = 1
ACT_NONE = 0
ACT_GELU_TANH = 1

EXPORTS = ("mxfp8_status_str", "mxfp8_scale_bytes", "mxfp8_quantize", "mxfp8_quantize_weight_f32",
           "mxfp8_linear_workspace_bytes", "mxfp8_linear", "mxfp8_gemm_prequant",
           "mxfp8_gelu_tanh_bf16", "mxfp8_device_status", "mxfp8_linear_noalloc",
           "mxfp8_gemm_quantize_out", "mxfp8_selftest_wait_timeout",
           "fp8rw_quantize_bf16", "fp8rw_quantize_weight_f32", "fp8rw_gemm", "fp8rw_linear_workspace_bytes",
           "fp8rw_linear",
           "nvfp4_scale_bytes", "nvfp4_amax_bf16", "nvfp4_amax_f32", "nvfp4_global_scale_from_amax",
           "nvfp4_quantize_bf16",
           "nvfp4_quantize_weight_f32", "nvfp4_gemm", "nvfp4_linear_workspace_bytes", "nvfp4_linear")


class MXFP8Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {_lib.mxfp8_status_str(status).decode()}")


def _check(status, where):
    if status != 0:
        raise MXFP8Error(status, where)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    """Device address of a CUDA tensor of the current device (None -> NULL).
    Every tensor handed to the library passes here, so host tensors and
    tensors of another device are refused before a kernel could be given
    their addresses."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(t.data_ptr())


def _cuda(t, name, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def scale_bytes(rows: int, K: int, layout: int = SF_TCGEN05) -> int:
    return int(_lib.mxfp8_scale_bytes(rows, K, layout))


def linear_workspace_bytes(M: int, K: int) -> int:
    return int(_lib.mxfp8_linear_workspace_bytes(M, K))


def quantize(x: torch.Tensor, layout: int = SF_TCGEN05, codes=None, scales=None):
    """BF16 [M, K] -> (E4M3 codes uint8 [M, K], E8M0 scales uint8 [bytes]).
    x may be a row-strided view (unit column stride, row stride >= K), e.g.
    a column slice of a fused projection's output."""
    if not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D BF16 CUDA tensor")
    M, K = x.shape
    ldx = x.stride(0) if M > 1 else K
    if x.stride(1) != 1 or ldx < K:
        raise ValueError("x must have unit column stride and row stride >= K")
    if codes is None:
        codes = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(scale_bytes(M, K, layout), 1), dtype=torch.uint8, device=x.device)
    _check(_lib.mxfp8_quantize(_ptr(x), M, K, ldx, _ptr(codes), _ptr(scales), layout, _stream()),
           "mxfp8_quantize")
    return codes, scales


def quantize_weight(w: torch.Tensor, layout: int = SF_TCGEN05):
    """FP32 [N, K] -> (E4M3 codes uint8 [N, K], E8M0 scales uint8 [bytes])."""
    _cuda(w, "w", torch.float32)
    N, K = w.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    scales = torch.empty(max(scale_bytes(N, K, layout), 1), dtype=torch.uint8, device=w.device)
    _check(_lib.mxfp8_quantize_weight_f32(_ptr(w), N, K, _ptr(codes), _ptr(scales), layout, _stream()),
           "mxfp8_quantize_weight_f32")
    return codes, scales


def linear(x: torch.Tensor, wq: torch.Tensor, wscale: torch.Tensor, bias=None, out=None, workspace=None):
    """Y = BF16(MXFP8(x) . MXFP8(W)^T + bias): x BF16 [M, K], wq [N, K], bias F16 [N]."""
    _cuda(x, "x", torch.bfloat16)
    _cuda(wq, "wq", torch.uint8)
    _cuda(wscale, "wscale", torch.uint8)
    M, K = x.shape
    N = wq.shape[0]
    if bias is not None:
        _cuda(bias, "bias", torch.float16)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = linear_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=x.device)
    _check(_lib.mxfp8_linear(_ptr(x), M, K, _ptr(wq), _ptr(wscale), N, _ptr(bias), _ptr(out),
                             _ptr(workspace), workspace.numel(), _stream()), "mxfp8_linear")
    return out


def linear_noalloc(x: torch.Tensor, wq: torch.Tensor, wscale: torch.Tensor, bias=None, out=None):
    """As `linear`, for callers that cannot allocate device memory: the
    library's fixed internal scratch replaces the workspace (M * K must fit
    32 MiB).  Only `out` is allocated here, and only when it is not given."""
    _cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(_lib.mxfp8_linear_noalloc(_ptr(x), M, K, _ptr(wq), _ptr(wscale), N, _ptr(bias), _ptr(out),
                                     _stream()), "mxfp8_linear_noalloc")
    return out


def gemm_prequant(xq, xscale, wq, wscale, bias=None, out=None):
    """Y from operands already quantized (tensor-core scale layout)."""
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _check(_lib.mxfp8_gemm_prequant(_ptr(xq), _ptr(xscale), M, K, _ptr(wq), _ptr(wscale), N,
                                    _ptr(bias), _ptr(out), _stream()), "mxfp8_gemm_prequant")
    return out


def gemm_quantize_out(xq, xscale, wq, wscale, bias=None, act=ACT_NONE, codes=None, scales=None):
    """The next linear's quantized input straight from this linear's GEMM:
    (E4M3 codes uint8 [M, N], tensor-core scales) of BF16(act(BF16(acc + bias)))
    without writing the BF16 output (act: ACT_NONE or ACT_GELU_TANH)."""
    M, K = xq.shape
    N = wq.shape[0]
    if codes is None:
        codes = torch.empty((M, N), dtype=torch.uint8, device=xq.device)
    if scales is None:
        scales = torch.empty(max(scale_bytes(M, N), 1), dtype=torch.uint8, device=xq.device)
    _check(_lib.mxfp8_gemm_quantize_out(_ptr(xq), _ptr(xscale), M, K, _ptr(wq), _ptr(wscale), N, _ptr(bias),
                                        act, _ptr(codes), _ptr(scales), _stream()), "mxfp8_gemm_quantize_out")
    return codes, scales


def gelu_tanh(x: torch.Tensor, out=None):
    _cuda(x, "x", torch.bfloat16)
    if out is None:
        out = torch.empty_like(x)
    _check(_lib.mxfp8_gelu_tanh_bf16(_ptr(x), _ptr(out), x.numel(), _stream()), "mxfp8_gelu_tanh_bf16")
    return out


# ------------------------------------------------------ per-channel FP8
def fp8rw_quantize(x: torch.Tensor, codes=None, scales=None):
    """BF16 [M, K] -> (E4M3 codes uint8 [M, K], FP32 scales [M]): one scale
    amax / 448 per row (token).  x may be a row-strided view."""
    if not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D BF16 CUDA tensor")
    M, K = x.shape
    ldx = x.stride(0) if M > 1 else K
    if x.stride(1) != 1 or ldx < K:
        raise ValueError("x must have unit column stride and row stride >= K")
    if codes is None:
        codes = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(_lib.fp8rw_quantize_bf16(_ptr(x), M, K, ldx, _ptr(codes), _ptr(scales), _stream()),
           "fp8rw_quantize_bf16")
    return codes, scales


def fp8rw_quantize_weight(w: torch.Tensor):
    """FP32 [N, K] -> (E4M3 codes uint8 [N, K], FP32 scales [N]), one per output channel."""
    _cuda(w, "w", torch.float32)
    N, K = w.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    scales = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(_lib.fp8rw_quantize_weight_f32(_ptr(w), N, K, _ptr(codes), _ptr(scales), _stream()),
           "fp8rw_quantize_weight_f32")
    return codes, scales


def fp8rw_gemm(xq, xscale, wq, wscale, bias=None, out=None):
    """Y = BF16(sx sw (Xq . Wq^T) + bias) from per-channel FP8 operands."""
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _check(_lib.fp8rw_gemm(_ptr(xq), _ptr(xscale), M, K, _ptr(wq), _ptr(wscale), N, _ptr(bias), _ptr(out),
                           _stream()), "fp8rw_gemm")
    return out


def fp8rw_linear_workspace_bytes(M: int, K: int) -> int:
    return int(_lib.fp8rw_linear_workspace_bytes(M, K))


def fp8rw_linear(x: torch.Tensor, wq, wscale, bias=None, out=None, workspace=None):
    """The per-channel FP8 layer: quantize x per token, then fp8rw_gemm."""
    _cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(fp8rw_linear_workspace_bytes(M, K), 256), dtype=torch.uint8, device=x.device)
    _check(_lib.fp8rw_linear(_ptr(x), M, K, _ptr(wq), _ptr(wscale), N, _ptr(bias), _ptr(out), _ptr(workspace),
                             workspace.numel(), _stream()), "fp8rw_linear")
    return out


# ---------------------------------------------------------------- NVFP4
def nvfp4_scale_bytes(rows: int, K: int) -> int:
    return int(_lib.nvfp4_scale_bytes(rows, K))


def nvfp4_amax(t: torch.Tensor) -> torch.Tensor:
    """amax of a contiguous BF16 or FP32 tensor (FP32 measured after
    rounding to BF16), as a 1-element FP32 CUDA tensor."""
    if not t.is_cuda or not t.is_contiguous() or t.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("t must be a contiguous BF16 or FP32 CUDA tensor")
    out = torch.empty(1, dtype=torch.float32, device=t.device)
    f = _lib.nvfp4_amax_bf16 if t.dtype == torch.bfloat16 else _lib.nvfp4_amax_f32
    _check(f(_ptr(t), t.numel(), _ptr(out), _stream()), "nvfp4_amax")
    return out


def nvfp4_global_scale(t: torch.Tensor) -> torch.Tensor:
    """The tensor's global scale RN(448 * 6 / amax) (1 for an all-zero
    tensor), computed on the device: a 1-element FP32 CUDA tensor."""
    amax = nvfp4_amax(t)
    g = torch.empty(1, dtype=torch.float32, device=t.device)
    _check(_lib.nvfp4_global_scale_from_amax(_ptr(amax), _ptr(g), _stream()), "nvfp4_global_scale_from_amax")
    return g


def _scale_tensor(g: torch.Tensor, what: str):
    if not isinstance(g, torch.Tensor):
        raise ValueError(f"{what} must be a 1-element FP32 CUDA tensor")
    _cuda(g, what, torch.float32)
    if g.numel() != 1:
        raise ValueError(f"{what} must hold one FP32 value (a global scale)")


def nvfp4_quantize(x: torch.Tensor, global_scale: torch.Tensor, codes=None, scales=None):
    """BF16 [M, K] -> (packed E2M1 codes uint8 [M, K/2], UE4M3 scales, tensor-core
    layout) with the global scale held in a 1-element FP32 CUDA tensor."""
    if not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D BF16 CUDA tensor")
    _scale_tensor(global_scale, "global_scale")
    M, K = x.shape
    ldx = x.stride(0) if M > 1 else K
    if x.stride(1) != 1 or ldx < K:
        raise ValueError("x must have unit column stride and row stride >= K")
    if codes is None:
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(nvfp4_scale_bytes(M, K), 1), dtype=torch.uint8, device=x.device)
    _check(_lib.nvfp4_quantize_bf16(_ptr(x), M, K, ldx, _ptr(global_scale), _ptr(codes), _ptr(scales),
                                    _stream()), "nvfp4_quantize_bf16")
    return codes, scales


def nvfp4_quantize_weight(w: torch.Tensor, global_scale: torch.Tensor):
    """FP32 [N, K] (rounded to BF16 first) -> (packed codes [N, K/2], scales)."""
    _cuda(w, "w", torch.float32)
    _scale_tensor(global_scale, "global_scale")
    N, K = w.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty(max(nvfp4_scale_bytes(N, K), 1), dtype=torch.uint8, device=w.device)
    _check(_lib.nvfp4_quantize_weight_f32(_ptr(w), N, K, _ptr(global_scale), _ptr(codes), _ptr(scales),
                                          _stream()), "nvfp4_quantize_weight_f32")
    return codes, scales


def nvfp4_gemm(xq, xscale, wq, wscale, x_global_scale: torch.Tensor, w_global_scale: torch.Tensor, bias=None,
               out=None):
    """Y = BF16(alpha sum_k (qx dec(sx)) (qw dec(sw)) + bias) from NVFP4
    operands: packed codes [M, K/2] / [N, K/2], their scales, and the two
    global scales (1-element FP32 CUDA tensors; the kernel forms alpha)."""
    _scale_tensor(x_global_scale, "x_global_scale")
    _scale_tensor(w_global_scale, "w_global_scale")
    M, K2 = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _check(_lib.nvfp4_gemm(_ptr(xq), _ptr(xscale), M, 2 * K2, _ptr(wq), _ptr(wscale), N, _ptr(x_global_scale),
                           _ptr(w_global_scale), _ptr(bias), _ptr(out), _stream()), "nvfp4_gemm")
    return out


def nvfp4_linear_workspace_bytes(M: int, K: int) -> int:
    return int(_lib.nvfp4_linear_workspace_bytes(M, K))


def nvfp4_linear(x: torch.Tensor, x_global_scale: torch.Tensor, wq, wscale, w_global_scale: torch.Tensor, bias=None,
                 out=None, workspace=None):
    """The NVFP4 layer: quantize x with its global scale, then nvfp4_gemm."""
    _cuda(x, "x", torch.bfloat16)
    _scale_tensor(x_global_scale, "x_global_scale")
    _scale_tensor(w_global_scale, "w_global_scale")
    M, K = x.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(nvfp4_linear_workspace_bytes(M, K), 256), dtype=torch.uint8, device=x.device)
    _check(_lib.nvfp4_linear(_ptr(x), M, K, _ptr(x_global_scale), _ptr(wq), _ptr(wscale), N, _ptr(w_global_scale),
                             _ptr(bias), _ptr(out), _ptr(workspace), workspace.numel(), _stream()), "nvfp4_linear")
    return out


SELFTEST_GEMM, SELFTEST_NVFP4_GEMM, SELFTEST_ROWWISE_QUANT = 0, 1, 2


def selftest_wait_timeout(which: int, timeout_ns: int) -> None:
    """Launch the bounded-wait self-test of one kernel family: the next
    device_status() reports MXFP8_ERR_TIMEOUT."""
    _check(_lib.mxfp8_selftest_wait_timeout(which, timeout_ns, _stream()), "mxfp8_selftest_wait_timeout")


def device_status() -> int:
    """Synchronize the current stream; 0 or the status a kernel recorded."""
    return int(_lib.mxfp8_device_status(_stream()))
