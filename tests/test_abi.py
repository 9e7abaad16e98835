"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wbmm.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"WBMM_API\s+[\w\s\*]+?\b(wbmm_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    # by path: the package's __init__ refuses to import before the library exists
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_wbmm_build", os.path.join(ROOT, "windowed_matmul_conv_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    return ctypes.CDLL(build.build())


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("wbmm_forward", "wbmm_backward", "wbmm_backward_workspace_bytes",
                     "wbmm_cache_matrices", "wbmm_forward_cached", "wbmm_dw3x3"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_binding_mirrors_the_header(lib):
    import windowed_matmul_conv_b200 as wb
    assert sorted(wb.EXPORTS) == sorted(declared_symbols())
    for name in wb.EXPORTS:
        assert callable(getattr(wb, name))


def _fwd(lib, x, T, y, B, C, H, W, w, dt):
    f = lib.wbmm_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    return f(x, T, y, B, C, H, W, w, dt, None)


def test_argument_checks_need_no_device(lib):
    a, b, c = 0x10000, 0x20000000, 0x40000000       # never dereferenced
    assert _fwd(lib, None, b, c, 1, 1, 14, 14, 7, 1) == 1   # null input
    assert _fwd(lib, a, b, c, 1, 1, 14, 15, 7, 1) == 2      # W % w
    assert _fwd(lib, a, b, c, 0, 1, 14, 14, 7, 1) == 1      # B = 0
    assert _fwd(lib, a, b, c, 1, 1, 14, 14, 7, 9) == 3      # dtype
    assert _fwd(lib, a + 2, b, c, 1, 1, 14, 14, 7, 1) == 4  # bf16 needs 16 B
    assert _fwd(lib, a, b, a + 64, 1, 1, 14, 14, 7, 1) == 1  # y overlaps x
    assert _fwd(lib, a, b, c, 1, 1, 130, 130, 65, 1) == 5   # w beyond limit


def test_workspace_size_formula(lib):
    f = lib.wbmm_backward_workspace_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int] * 6
    # bf16, tensor-core path: one partial table per (channel, CTA range)
    # segment, at most n = C + min(256, tiles) - 1 of them, then one 64-bit
    # flag per table (8-byte aligned).
    def tc(n, tsz=729):
        return ((n * tsz + 1) // 2 * 2 + 2 * n) * 4
    # training workload: 64-window tiles of 32 two-window bands, 8 tiles per
    # channel, 2048 tiles -> 256 + 255 tables
    assert f(128, 256, 28, 28, 14, 1) == tc(256 + 255)
    # 64 images of 56x56: 16 bands/tile, 16 tiles/channel, 2048 tiles
    assert f(64, 128, 56, 56, 14, 1) == tc(128 + 255)
    # 32 images of 112x112: 8 bands/tile, 32 tiles/channel, 128 tiles
    assert f(32, 4, 112, 112, 14, 1) == tc(4 + 127)
    # 2 images of 112x112, w = 7: 64-window tiles of 4 bands, 8 tiles/channel
    assert f(2, 4, 112, 112, 7, 1) == tc(4 + 31, 169)
    # fp32, CUDA-core path: chunks of 8 bands per channel
    assert f(2, 3, 14, 28, 7, 0) == 3 * 1 * 169 * 4
    assert f(1, 1, 14, 15, 7, 1) == 0


def test_status_strings(lib):
    f = lib.wbmm_status_string
    f.restype = ctypes.c_char_p
    f.argtypes = [ctypes.c_int]
    for s in range(9):
        assert f(s).decode().startswith("WBMM_")
