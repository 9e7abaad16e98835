"""The CUDA-core table gradient's partial-table slots, without a GPU.

For 4 <= w <= 14 the fp32 table gradient splits all channels' tiles (whole
bands, at most 64 windows) into one contiguous, balanced range per block
and writes one partial table per (channel, block that touches it).  The
workspace the library reports must hold a slot for every such block: here
the ranges are enumerated by brute force, with the grid the library plans
(148 SMs times the blocks that fit one SM), and the number of blocks that
touch each channel is compared with the slots the workspace size implies.
"""
import ctypes
import os
import random

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COUNTER_WORDS = 65536
SMS = 148
TILE_WINDOWS = 64
MAX_COLS = TILE_WINDOWS * 14
MAX_THREADS = 640


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_wbmm_build", os.path.join(ROOT, "windowed_matmul_conv_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    f = ctypes.CDLL(build.build()).wbmm_backward_workspace_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int] * 6
    return f


def planned_grid(C, ntiles, w, W):
    """Blocks of the launch: 148 x the blocks one SM holds (shared memory,
    threads and registers), at most one per tile."""
    d = w * w
    dp = (d + 7) // 8 * 8
    ug = (d + 7) // 8
    threads = (ug * ug + 31) // 32 * 32
    smem = 4 * TILE_WINDOWS * dp * 4 + MAX_COLS * 4
    regs = 65536 // MAX_THREADS // 8 * 8
    bps = 233472 // (smem + 1024)
    bps = min(bps, 2048 // threads)
    bps = max(1, min(bps, 65536 // (threads * regs)))
    return min(C * ntiles, SMS * bps)


def blocks_per_channel(C, ntiles, grid):
    """Number of blocks whose range [b*T/G, (b+1)*T/G) meets each channel."""
    total = C * ntiles
    most = 0
    for c in range(C):
        first, last = c * ntiles, c * ntiles + ntiles - 1
        b_first = ((first + 1) * grid - 1) // total
        b_last = ((last + 1) * grid - 1) // total
        assert b_first * total // grid <= first < (b_first + 1) * total // grid
        most = max(most, b_last - b_first + 1)
    return most


def shapes(n):
    rng = random.Random(1234)
    for _ in range(n):
        w = rng.randint(4, 14)
        nh, nw = rng.randint(1, 6), rng.randint(1, 12)
        yield rng.randint(1, 48), rng.randint(1, 300), nh * w, nw * w, w


@pytest.mark.parametrize("shape", list(shapes(60)) + [(128, 256, 28, 28, 14), (3, 2, 56, 56, 7),
                                                     (1, 1, 14, 14, 14), (64, 1, 56, 896, 14)],
                         ids=lambda s: "x".join(map(str, s)))
def test_workspace_holds_every_block_of_a_channel(lib, shape):
    B, C, H, W, w = shape
    nh, nw = H // w, W // w
    tsz = (2 * w - 1) ** 2
    nbytes = lib(B, C, H, W, w, 0)           # fp32
    floats = nbytes // 4 - COUNTER_WORDS
    assert floats % (C * tsz) == 0
    slots = floats // (C * tsz)
    bpt = TILE_WINDOWS // nw
    ntiles = -(-(B * nh) // bpt)
    grid = planned_grid(C, ntiles, w, W)
    need = blocks_per_channel(C, ntiles, grid)
    assert need <= slots, (need, slots, grid, ntiles)
