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
    # bf16, tensor-core path: a fixed region of 65536 arrival counters, then
    # one partial table per (channel, CTA range) segment, at most
    # n = C + min(256, tiles) - 1 of them.
    def tc(C, grid, tsz=729):
        n = C + grid - 1
        return (65536 + n * tsz) * 4
    # training workload: 64-window tiles of 32 two-window bands, 8 tiles per
    # channel, 2048 tiles -> 256 + 255 tables
    assert f(128, 256, 28, 28, 14, 1) == tc(256, 256)
    # 64 images of 56x56: 16 bands/tile, 16 tiles/channel, 2048 tiles
    assert f(64, 128, 56, 56, 14, 1) == tc(128, 256)
    # 32 images of 112x112: 8 bands/tile, 32 tiles/channel, 128 tiles
    assert f(32, 4, 112, 112, 14, 1) == tc(4, 128)
    # 2 images of 112x112, w = 7: 64-window tiles of 4 bands, 8 tiles/channel
    assert f(2, 4, 112, 112, 7, 1) == tc(4, 32, 169)
    # fp32, CUDA-core path, 4 <= w <= 14: tiles of whole bands (at most 64
    # windows); all channels' tiles split into min(148, tiles) contiguous
    # ranges; a channel spans at most 2 + (n - 2) // (fewest tiles of a
    # range) of them (n tiles per channel, capped at n), one partial table
    # slot each
    assert f(2, 3, 14, 28, 7, 0) == (65536 + 3 * 1 * 169) * 4
    # training workload: 8 tiles per channel, 2048 tiles in ranges of 13 or 14
    assert f(128, 256, 28, 28, 14, 0) == (65536 + 256 * 2 * 729) * 4
    # 3 tiles per channel, 6 tiles, one per range: 3 slots
    assert f(3, 2, 56, 56, 7, 0) == (65536 + 2 * 3 * 169) * 4
    # w > 14: chunks of 8 bands per channel
    assert f(2, 3, 40, 40, 20, 0) == (65536 + 3 * 1 * 1521) * 4
    assert f(9, 1, 40, 40, 20, 0) == (65536 + 1 * 3 * 1521) * 4
    assert f(1, 1, 14, 15, 7, 1) == 0


def test_status_strings(lib):
    f = lib.wbmm_status_string
    f.restype = ctypes.c_char_p
    f.argtypes = [ctypes.c_int]
    for s in range(9):
        assert f(s).decode().startswith("WBMM_")


def _proto(lib, name, argtypes):
    f = getattr(lib, name)
    f.restype = ctypes.c_int
    f.argtypes = argtypes
    return f


P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

# Addresses that are never dereferenced: every call below must be rejected by
# the host-side checks, before any device call.  Blocks are 256 MB apart so
# that buffers of the shapes used never overlap unless a test says so.
A0, A1, A2, A3, A4 = (0x10000000 * k for k in (1, 2, 3, 4, 5))


def test_backward_argument_checks(lib):
    f = _proto(lib, "wbmm_backward", [P, P, P, P, P, P, S] + [I] * 6 + [P])
    ws = lib.wbmm_backward_workspace_bytes
    ws.restype, ws.argtypes = S, [I] * 6
    need = ws(2, 4, 28, 28, 14, 1)
    assert need > 0

    def call(x=A0, T=A1, dY=A2, dX=A3, dT=A4, work=A4 + 0x100000, nbytes=need,
             shape=(2, 4, 28, 28, 14), dt=1):
        return f(x, T, dY, dX, dT, work, nbytes, *shape, dt, None)

    assert call(dt=2) == 3                               # dtype
    assert call(dY=None) == 1                            # dY is required
    assert call(T=None) == 1                             # dX needs the table
    assert call(x=None) == 1                             # dT needs the input
    assert call(shape=(2, 4, 28, 30, 14)) == 2           # W % w
    assert call(shape=(2, 4, 28, 28, 0)) == 1            # w = 0
    assert call(shape=(2, 4, 130, 130, 65)) == 5         # w beyond limit
    assert call(dX=A3 + 8) == 4                          # bf16 maps need 16 B
    assert call(dT=A4 + 2) == 4                          # dT is fp32
    assert call(dX=A2 + 64) == 1                         # dX overlaps dY
    assert call(dT=A0 + 64) == 1                         # dT overlaps x
    assert call(work=None) == 6                          # dT needs a workspace
    assert call(nbytes=need - 4) == 6                    # ... of the stated size
    assert call(work=A4 + 0x100008) == 4                 # ... 16-byte aligned
    assert call(work=A4 + 64) == 1                       # ... not overlapping dT
    assert call(work=A2 + 64) == 1                       # ... nor dY
    # dX only: neither x nor a workspace is needed, so the first failing check
    # is the misaligned dX
    assert call(dT=None, x=None, work=None, nbytes=0, dX=A3 + 8) == 4
    # dT only: no table needed
    assert call(dX=None, T=None, dT=A4 + 2) == 4


def test_cache_and_merge_argument_checks(lib):
    cache = _proto(lib, "wbmm_cache_matrices", [P, P, I, I, I, P])
    assert cache(A0, A1, 4, 14, 3, None) == 3
    assert cache(None, A1, 4, 14, 1, None) == 1
    assert cache(A0, A1, 0, 14, 1, None) == 1
    assert cache(A0, A1, 4, 65, 1, None) == 5
    assert cache(A0, A1 + 2, 4, 14, 1, None) == 4
    assert cache(A0, A0 + 128, 4, 14, 1, None) == 1      # M overlaps T
    merge = _proto(lib, "wbmm_reparam_merge", [P, P, P, I, I, I, I, P])
    assert merge(A0, A1, A2, 4, 14, 7, 5, None) == 3
    assert merge(A0, None, A2, 4, 14, 7, 1, None) == 1
    assert merge(A0, A1, A2, 4, 14, 5, 1, None) == 1     # k must divide w
    assert merge(A0, A1, A2, 4, 14, 0, 1, None) == 1
    assert merge(A0, A1, A2, 4, 70, 7, 1, None) == 5
    assert merge(A0, A1, A2 + 8, 4, 14, 7, 1, None) == 4
    assert merge(A0, A2 + 64, A2, 4, 14, 7, 1, None) == 1  # M overlaps the small table


def test_cached_and_dw_argument_checks(lib):
    fc = _proto(lib, "wbmm_forward_cached", [P, P, P, P] + [I] * 6 + [P])
    assert fc(A0, A1, None, A2, 1, 4, 28, 28, 14, 4, None) == 3
    assert fc(A0, None, None, A2, 1, 4, 28, 28, 14, 1, None) == 1
    assert fc(A0, A1, None, A2, 1, 4, 28, 21, 14, 1, None) == 2
    assert fc(A0, A1, A3 + 2, A2, 1, 4, 28, 28, 14, 1, None) == 4   # 3x3 weights
    assert fc(A0, A1, None, A0 + 16, 1, 4, 28, 28, 14, 1, None) == 1  # out overlaps x
    assert fc(A0, A1, A2 + 16, A2, 1, 4, 28, 28, 14, 1, None) == 1  # out overlaps the weights
    dw = _proto(lib, "wbmm_dw3x3", [P, P, P] + [I] * 5 + [P])
    assert dw(A0, A1, A2, 1, 4, 9, 13, 7, None) == 3
    assert dw(A0, A1, None, 1, 4, 9, 13, 1, None) == 1
    assert dw(A0, A1, A2, 1, 4, 0, 13, 1, None) == 1
    assert dw(A0 + 8, A1, A2, 1, 4, 9, 13, 1, None) == 4
    assert dw(A0, A1, A0 + 32, 1, 4, 9, 13, 1, None) == 1           # in place is refused


def test_static_table_gradient_argument_checks(lib):
    f = _proto(lib, "wbmm_backward_dt_static", [P, P, P] + [I] * 6 + [P])
    assert f(A0, A1, A2, 2, 4, 28, 28, 14, 2, None) == 3
    assert f(A0, None, A2, 2, 4, 28, 28, 14, 1, None) == 1
    assert f(A0, A1, A2, 2, 4, 28, 27, 14, 1, None) == 2
    assert f(A0, A1, A2, 2, 4, 130, 130, 65, 1, None) == 5
    assert f(A0, A1 + 8, A2, 2, 4, 28, 28, 14, 1, None) == 4
    assert f(A0, A1, A0 + 64, 2, 4, 28, 28, 14, 1, None) == 1       # dT overlaps x
    # more partial tables than the 4 MiB static array holds
    assert f(A0, A1, A2, 1, 2048, 14, 14, 14, 1, None) == 6
