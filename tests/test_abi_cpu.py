"""The C-ABI library loads and exports every symbol include/*.h declares;
host-side argument checks reject bad calls before anything is launched.
No GPU needed: none of these calls reaches the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PREFIXES = ("mxfp8_", "fp8rw_", "nvfp4_")


def declared_functions():
    names = set()
    for h in sorted(os.listdir(INCLUDE)):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(INCLUDE, h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b((?:%s)[a-z0-9_]+)\s*\(" % "|".join(PREFIXES), text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from mxfp8_w8a8_quantized_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("mxfp8_quantize", "mxfp8_linear", "mxfp8_quantize_weight_f32", "mxfp8_gemm_prequant",
                 "mxfp8_scale_bytes", "mxfp8_linear_workspace_bytes", "mxfp8_status_str",
                 "mxfp8_gelu_tanh_bf16", "mxfp8_device_status"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_binding_exports_match_header():
    from mxfp8_w8a8_quantized_b200 import mxfp8
    assert sorted(mxfp8.EXPORTS) == [n for n in declared_functions() if n in mxfp8.EXPORTS]
    assert set(declared_functions()) <= set(mxfp8.EXPORTS) | set()


def _sig(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.mxfp8_scale_bytes.argtypes = [I64, I64, ctypes.c_int]
    lib.mxfp8_scale_bytes.restype = ctypes.c_size_t
    lib.mxfp8_linear_workspace_bytes.argtypes = [I64, I64]
    lib.mxfp8_linear_workspace_bytes.restype = ctypes.c_size_t
    lib.mxfp8_quantize.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, P]
    lib.mxfp8_quantize_weight_f32.argtypes = [P, I64, I64, P, P, ctypes.c_int, P]
    lib.mxfp8_linear.argtypes = [P, I64, I64, P, P, I64, P, P, P, ctypes.c_size_t, P]
    lib.mxfp8_gemm_prequant.argtypes = [P, P, I64, I64, P, P, I64, P, P, P]
    lib.mxfp8_gelu_tanh_bf16.argtypes = [P, P, I64, P]
    lib.mxfp8_status_str.argtypes = [ctypes.c_int]
    lib.mxfp8_status_str.restype = ctypes.c_char_p
    return lib


def test_sizes(lib):
    L = _sig(lib)
    assert L.mxfp8_scale_bytes(256, 512, 0) == 256 * 16
    assert L.mxfp8_scale_bytes(256, 512, 1) == 2 * 4 * 512
    assert L.mxfp8_scale_bytes(32760, 5120, 1) == 256 * 40 * 512   # ceil(32760/128) = 256
    assert L.mxfp8_scale_bytes(1, 32, 1) == 512                    # padded to one atom
    assert L.mxfp8_scale_bytes(10, 33, 1) == 0                     # K % 32 != 0
    assert L.mxfp8_scale_bytes(-1, 32, 0) == 0
    assert L.mxfp8_scale_bytes(10, 32, 7) == 0
    ws = L.mxfp8_linear_workspace_bytes(32760, 5120)
    assert ws == 32760 * 5120 + 256 * 40 * 512


def test_status_strings(lib):
    L = _sig(lib)
    for s in range(6):
        assert L.mxfp8_status_str(s).startswith(b"MXFP8_")
    assert b"UNKNOWN" in L.mxfp8_status_str(99)


FAKE = 0x10000  # a 16-byte aligned, never dereferenced address


def test_argument_checks_return_before_launch(lib):
    L = _sig(lib)
    ARG, ALIGN, SHAPE = 1, 2, 3
    # quantize
    assert L.mxfp8_quantize(None, 4, 64, 64, FAKE, FAKE, 1, None) == ARG
    assert L.mxfp8_quantize(FAKE, 4, 48, 48, FAKE, FAKE, 1, None) == SHAPE      # K % 32
    assert L.mxfp8_quantize(FAKE, 4, 64, 32, FAKE, FAKE, 1, None) == ARG        # ldx < K
    assert L.mxfp8_quantize(FAKE + 2, 4, 64, 64, FAKE, FAKE, 1, None) == ALIGN  # X misaligned
    assert L.mxfp8_quantize(FAKE, 4, 64, 68, FAKE, FAKE, 1, None) == ALIGN      # row stride
    assert L.mxfp8_quantize(FAKE, 4, 64, 64, FAKE, FAKE, 5, None) == ARG        # layout
    assert L.mxfp8_quantize(FAKE, -1, 64, 64, FAKE, FAKE, 1, None) == ARG
    assert L.mxfp8_quantize(FAKE, 0, 64, 64, FAKE, FAKE, 1, None) == 0          # empty: no-op
    # weights
    assert L.mxfp8_quantize_weight_f32(FAKE, 4, 40, FAKE, FAKE, 1, None) == SHAPE
    # gemm
    assert L.mxfp8_gemm_prequant(FAKE, FAKE, 4, 96, FAKE, FAKE, 16, None, FAKE, None) == SHAPE   # K % 128
    assert L.mxfp8_gemm_prequant(FAKE, FAKE, 4, 128, FAKE, FAKE, 12, None, FAKE, None) == SHAPE  # N % 8
    assert L.mxfp8_gemm_prequant(FAKE, FAKE, 4, 128, FAKE, FAKE, 16, FAKE + 8, FAKE, None) == ALIGN
    assert L.mxfp8_gemm_prequant(FAKE, None, 4, 128, FAKE, FAKE, 16, None, FAKE, None) == ARG
    assert L.mxfp8_gemm_prequant(FAKE, FAKE, 0, 128, FAKE, FAKE, 16, None, FAKE, None) == 0
    assert L.mxfp8_gemm_prequant(FAKE, FAKE, 4, 128, FAKE, FAKE, 0, None, FAKE, None) == ARG
    # linear: workspace too small, misaligned workspace
    need = L.mxfp8_linear_workspace_bytes(4, 128)
    assert L.mxfp8_linear(FAKE, 4, 128, FAKE, FAKE, 16, None, FAKE, FAKE, need - 1, None) == ARG
    assert L.mxfp8_linear(FAKE, 4, 128, FAKE, FAKE, 16, None, FAKE, FAKE + 16, need, None) == ALIGN
    assert L.mxfp8_linear(FAKE, 4, 100, FAKE, FAKE, 16, None, FAKE, FAKE, 1 << 20, None) == SHAPE
    # gelu
    assert L.mxfp8_gelu_tanh_bf16(FAKE, FAKE, 12, None) == SHAPE
    assert L.mxfp8_gelu_tanh_bf16(FAKE, FAKE + 4, 16, None) == ALIGN
    assert L.mxfp8_gelu_tanh_bf16(FAKE, FAKE, 0, None) == 0


def test_fp8_rowwise_argument_checks_return_before_launch(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.fp8rw_quantize_bf16.argtypes = [P, I64, I64, I64, P, P, P]
    lib.fp8rw_quantize_weight_f32.argtypes = [P, I64, I64, P, P, P]
    lib.fp8rw_gemm.argtypes = [P, P, I64, I64, P, P, I64, P, P, P]
    lib.fp8rw_linear_workspace_bytes.argtypes = [I64, I64]
    lib.fp8rw_linear_workspace_bytes.restype = ctypes.c_size_t
    lib.fp8rw_linear.argtypes = [P, I64, I64, P, P, I64, P, P, P, ctypes.c_size_t, P]
    L = lib
    ARG, ALIGN, SHAPE = 1, 2, 3
    assert L.fp8rw_quantize_bf16(FAKE, 4, 60, 60, FAKE, FAKE, None) == SHAPE         # K % 8
    assert L.fp8rw_quantize_bf16(FAKE, 4, 16392, 16392, FAKE, FAKE, None) == SHAPE   # K > 16384
    assert L.fp8rw_quantize_bf16(FAKE, 4, 64, 60, FAKE, FAKE, None) == ARG           # ldx < K
    assert L.fp8rw_quantize_bf16(FAKE, 4, 64, 68, FAKE, FAKE, None) == ALIGN         # row stride
    assert L.fp8rw_quantize_bf16(FAKE, 4, 64, 64, FAKE, FAKE + 2, None) == ALIGN     # scales
    assert L.fp8rw_quantize_bf16(None, 4, 64, 64, FAKE, FAKE, None) == ARG
    assert L.fp8rw_quantize_bf16(FAKE, 0, 64, 64, FAKE, FAKE, None) == 0
    assert L.fp8rw_quantize_weight_f32(FAKE, 4, 66, FAKE, FAKE, None) == SHAPE      # K % 4
    assert L.fp8rw_quantize_weight_f32(FAKE + 4, 4, 64, FAKE, FAKE, None) == ALIGN
    assert L.fp8rw_gemm(FAKE, FAKE, 4, 96, FAKE, FAKE, 16, None, FAKE, None) == SHAPE
    assert L.fp8rw_gemm(FAKE, FAKE + 4, 4, 128, FAKE, FAKE, 16, None, FAKE, None) == ALIGN
    assert L.fp8rw_gemm(FAKE, FAKE, 0, 128, FAKE, FAKE, 16, None, FAKE, None) == 0
    need = L.fp8rw_linear_workspace_bytes(4, 128)
    assert need == 512 + 16
    assert L.fp8rw_linear(FAKE, 4, 128, FAKE, FAKE, 16, None, FAKE, FAKE, need - 1, None) == ARG
    assert L.fp8rw_linear(FAKE, 4, 128, FAKE, FAKE, 16, None, FAKE, FAKE + 16, need, None) == ALIGN


def test_nvfp4_gemm_argument_checks_return_before_launch(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.nvfp4_gemm.argtypes = [P, P, I64, I64, P, P, I64, P, P, P, P, P]
    lib.nvfp4_linear_workspace_bytes.argtypes = [I64, I64]
    lib.nvfp4_linear_workspace_bytes.restype = ctypes.c_size_t
    lib.nvfp4_linear.argtypes = [P, I64, I64, P, P, P, I64, P, P, P, P, ctypes.c_size_t, P]
    lib.nvfp4_global_scale_from_amax.argtypes = [P, P, P]
    lib.nvfp4_quantize_bf16.argtypes = [P, I64, I64, I64, P, P, P, P]
    L = lib
    ARG, ALIGN, SHAPE = 1, 2, 3
    G = FAKE                                     # a device float holding a global scale
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 96, FAKE, FAKE, 16, G, G, None, FAKE, None) == SHAPE    # K % 64
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 128, FAKE, FAKE, 12, G, G, None, FAKE, None) == SHAPE   # N % 8
    assert L.nvfp4_gemm(FAKE, FAKE + 4, 4, 128, FAKE, FAKE, 16, G, G, None, FAKE, None) == ALIGN
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 128, FAKE, FAKE, 16, G, G, FAKE + 2, FAKE, None) == ALIGN  # bias
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 128, FAKE, FAKE, 16, None, G, None, FAKE, None) == ARG     # g_x
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 128, FAKE, FAKE, 16, G, None, None, FAKE, None) == ARG     # g_w
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 128, FAKE, FAKE, 16, G + 2, G, None, FAKE, None) == ALIGN  # float alignment
    assert L.nvfp4_gemm(FAKE, FAKE, 4, 128, FAKE, None, 16, G, G, None, FAKE, None) == ARG
    assert L.nvfp4_gemm(FAKE, FAKE, 0, 128, FAKE, FAKE, 16, G, G, None, FAKE, None) == 0
    need = L.nvfp4_linear_workspace_bytes(4, 128)
    assert need == 256 + 2 * 512                 # codes rounded to 256 B + one row block of 2 scale atoms
    assert L.nvfp4_linear(FAKE, 4, 128, G, FAKE, FAKE, 16, G, None, FAKE, FAKE, need - 1, None) == ARG
    assert L.nvfp4_linear(FAKE, 4, 128, G, FAKE, FAKE, 16, G, None, FAKE, FAKE + 16, need, None) == ALIGN
    assert L.nvfp4_linear(FAKE, 4, 96, G, FAKE, FAKE, 16, G, None, FAKE, FAKE, need, None) == SHAPE
    assert L.nvfp4_linear(FAKE, 4, 128, None, FAKE, FAKE, 16, G, None, FAKE, FAKE, need, None) == ARG
    # the GEMM's own checks also run before the quantizer is launched (a
    # launch here would fail with a CUDA error, not these codes)
    assert L.nvfp4_linear(FAKE, 4, 128, G, FAKE, FAKE, 16, None, None, FAKE, FAKE, need, None) == ARG    # g_w
    assert L.nvfp4_linear(FAKE, 4, 128, G, FAKE, FAKE, 16, G, None, None, FAKE, need, None) == ARG       # Y
    assert L.nvfp4_linear(FAKE, 4, 128, G, FAKE + 4, FAKE, 16, G, None, FAKE, FAKE, need, None) == ALIGN
    assert L.nvfp4_linear(FAKE, 4, 128, G, FAKE, FAKE, 12, G, None, FAKE, FAKE, need, None) == SHAPE     # N % 8
    assert L.nvfp4_global_scale_from_amax(None, G, None) == ARG
    assert L.nvfp4_global_scale_from_amax(G, G + 1, None) == ALIGN
    assert L.nvfp4_quantize_bf16(FAKE, 4, 128, 128, None, FAKE, FAKE, None) == ARG                      # g
    assert L.nvfp4_quantize_bf16(FAKE, 4, 128, 128, G + 2, FAKE, FAKE, None) == ALIGN


def test_product_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib.util
    import sys
    src = os.path.join(ROOT, "mxfp8_w8a8_quantized_b200", "mxfp8.py")
    # load a copy of the binding next to no library: the import must raise
    dst = tmp_path / "mxfp8.py"
    dst.write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("mxfp8_copy", str(dst))
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
    assert "mxfp8_copy" not in sys.modules


def test_binding_checks_every_status_with_its_entry_name():
    """Each C call in the binding goes through _check(status, name), the
    name being the entry point called."""
    import ast
    src = open(os.path.join(ROOT, "mxfp8_w8a8_quantized_b200", "mxfp8.py")).read()
    calls = [n for n in ast.walk(ast.parse(src)) if isinstance(n, ast.Call) and getattr(n.func, "id", None) == "_check"]
    assert calls
    for c in calls:
        assert len(c.args) == 2, ast.unparse(c)[:120]
        status, name = c.args
        assert isinstance(status, ast.Call) and isinstance(name, ast.Constant)
        if isinstance(status.func, ast.Attribute):      # _lib.<entry>(...); else a chosen entry
            assert status.func.attr == name.value, ast.unparse(c)[:120]


def test_selftest_argument_checks(lib):
    P = ctypes.c_void_p
    lib.mxfp8_selftest_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_uint64, P]
    ARG = 1
    assert lib.mxfp8_selftest_wait_timeout(3, 1000000, None) == ARG          # unknown kernel family
    assert lib.mxfp8_selftest_wait_timeout(-1, 1000000, None) == ARG
    assert lib.mxfp8_selftest_wait_timeout(0, 0, None) == ARG                # no limit
    assert lib.mxfp8_selftest_wait_timeout(0, 20_000_000_000, None) == ARG   # above 10 s


def test_noalloc_rejects_before_launch(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.mxfp8_linear_noalloc.argtypes = [P, I64, I64, P, P, I64, P, P, P]
    ARG, ALIGN, SHAPE = 1, 2, 3
    L = lib
    assert L.mxfp8_linear_noalloc(FAKE, 4, 128, FAKE, FAKE, 12, None, FAKE, None) == SHAPE      # N % 8
    assert L.mxfp8_linear_noalloc(FAKE, 4, 96, FAKE, FAKE, 16, None, FAKE, None) == SHAPE       # K % 128
    assert L.mxfp8_linear_noalloc(FAKE, 4, 128, FAKE + 4, FAKE, 16, None, FAKE, None) == ALIGN  # Wq
    assert L.mxfp8_linear_noalloc(FAKE, 4, 128, FAKE, FAKE, 16, FAKE + 2, FAKE, None) == ALIGN  # bias
    assert L.mxfp8_linear_noalloc(FAKE, 4, 128, FAKE, FAKE, 16, None, None, None) == ARG        # Y
    assert L.mxfp8_linear_noalloc(FAKE, 1 << 20, 5120, FAKE, FAKE, 16, None, FAKE, None) == SHAPE  # scratch
    assert L.mxfp8_linear_noalloc(FAKE, 6554, 5120, FAKE, FAKE, 16, None, FAKE, None) == SHAPE     # codes cap + 1 row
    # codes fit (32 x 524416 B), the scales (4 x 524416 B > 2 MiB) do not
    assert L.mxfp8_linear_noalloc(FAKE, 32, (1 << 19) + 128, FAKE, FAKE, 16, None, FAKE, None) == SHAPE


def test_binding_refuses_host_tensors():
    """A host tensor never reaches the library: every wrapper raises
    ValueError before the C call (a kernel given a host address would
    fault)."""
    import torch
    from mxfp8_w8a8_quantized_b200 import mxfp8 as mx
    u8 = lambda *s: torch.zeros(*s, dtype=torch.uint8)
    f32 = lambda *s: torch.zeros(*s, dtype=torch.float32)
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    calls = [
        lambda: mx.quantize(bf(4, 128)),
        lambda: mx.quantize_weight(f32(8, 128)),
        lambda: mx.linear(bf(4, 128), u8(8, 128), u8(512)),
        lambda: mx.linear_noalloc(bf(4, 128), u8(8, 128), u8(512)),
        lambda: mx.gemm_prequant(u8(4, 128), u8(512), u8(8, 128), u8(512)),
        lambda: mx.gemm_quantize_out(u8(4, 128), u8(512), u8(128, 128), u8(512)),
        lambda: mx.gelu_tanh(bf(64)),
        lambda: mx.fp8rw_quantize(bf(4, 128)),
        lambda: mx.fp8rw_quantize_weight(f32(8, 128)),
        lambda: mx.fp8rw_gemm(u8(4, 128), f32(4), u8(8, 128), f32(8)),
        lambda: mx.fp8rw_linear(bf(4, 128), u8(8, 128), f32(8)),
        lambda: mx.nvfp4_amax(bf(64)),
        lambda: mx.nvfp4_global_scale(bf(64)),
        lambda: mx.nvfp4_quantize(bf(4, 128), f32(1)),
        lambda: mx.nvfp4_quantize_weight(f32(8, 128), f32(1)),
        lambda: mx.nvfp4_gemm(u8(4, 64), u8(1024), u8(8, 64), u8(1024), f32(1), f32(1)),
        lambda: mx.nvfp4_linear(bf(4, 128), f32(1), u8(8, 64), u8(1024), f32(1)),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(ValueError):
            call()
