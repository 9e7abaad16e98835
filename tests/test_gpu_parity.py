"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes span several tiles and a ragged last tile for every window size
class the tensor-core kernels compile (one and two 128-row M tiles, odd and
even w); the full-size workloads run in the launch configuration the
benchmark times and are compared on sampled (image, channel) planes, which
the oracle computes exactly because planes are independent.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import (check_bf16, check_f32, dt_bound, forward_rowbound, to_np,
                         window_norms)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import windowed_matmul_conv_b200 as wb  # noqa: E402

DEV = "cuda:0"


def gen(shape, seed, dtype=torch.bfloat16, scale=1.0):
    return synth.draw_tensor(shape, seed, "f32", scale).to(dtype).to(DEV)


def run_forward(x, T, w):
    y = wb.forward(x, T, w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    return y


# (B, C, H, W, w): several tiles and a ragged tail per shape
BF16_SHAPES = [
    (9, 3, 56, 56, 14),     # 36 bands/channel, 16-band tiles -> 16, 16, 4
    (2, 4, 42, 28, 14),     # nh = 3, nw = 2
    (5, 2, 105, 112, 7),    # one 128-row M tile, 128-window tiles, ragged
    (3, 3, 48, 64, 16),     # d = 256, no K padding
    (4, 2, 39, 104, 13),    # odd w with two M tiles
    (6, 3, 40, 40, 5),      # odd w, one M tile
    (3, 2, 24, 48, 3),
    (2, 2, 24, 96, 12),
]


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_forward_bf16_small(shape):
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 1)
    T = gen((C, (2 * w - 1) ** 2), 2, scale=0.02)
    y = run_forward(x, T, w)
    assert wb.wbmm_last_path() == 1, "tensor-core kernel expected"
    xr, Tr = to_np(x), to_np(T)
    ref = oracle.forward(xr, Tr, w)
    check_bf16(to_np(y), ref, forward_rowbound(xr, Tr, w), "forward")


# w = 28 on tensor cores (128 windows per tile as the MMA's M dimension in
# tensor memory, a Toeplitz stack of the table as B): one partial tile per
# channel (4, 18 or 15 bands of 32 or 64), one tile on each of 60 CTAs, and
# three tiles per channel on more tiles than CTAs, so that CTAs take two
# tiles, cross channel boundaries, rebuild the stack and hand the A rows
# from one tile to the next (checked on sampled channels)
BIG_SHAPES = [(2, 3, 56, 112, 28), (9, 2, 56, 112, 28), (5, 2, 84, 56, 28), (9, 60, 56, 112, 28),
              (40, 60, 56, 112, 28)]


@pytest.mark.parametrize("shape", BIG_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_w28_forward_and_dx_tensor_cores(shape):
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 33)
    dy = gen((B, C, H, W), 34)
    T = gen((C, (2 * w - 1) ** 2), 35, scale=0.02)
    y = run_forward(x, T, w)
    assert wb.wbmm_last_path() == 1, "tensor-core kernel expected"
    dX, _ = wb.backward(x, T, dy, w, need_dt=False)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    assert wb.wbmm_last_path() == 1
    cs = list(range(C)) if C <= 3 else [0, 1, C // 2, C - 2, C - 1]
    xr, gr, Tr = to_np(x[:, cs]), to_np(dy[:, cs]), to_np(T[cs])
    check_bf16(to_np(y[:, cs]), oracle.forward(xr, Tr, w), forward_rowbound(xr, Tr, w), "w28 y")
    check_bf16(to_np(dX[:, cs]), oracle.backward_dx(gr, Tr, w),
               forward_rowbound(gr, Tr[:, ::-1].copy(), w), "w28 dX")


def test_forward_fp32_tiny_workload():
    wl = synth.WORKLOADS["tiny_fp32"]
    d = synth.draw(wl, seed=0)
    x, T = d["x"].to(DEV), d["T"].to(DEV)
    y = run_forward(x, T, wl.w)
    ref = oracle.forward(d["x"], d["T"], wl.w)
    absdot = oracle.forward(np.abs(to_np(d["x"])), np.abs(to_np(d["T"])), wl.w)
    check_f32(to_np(y), ref, absdot, "tiny fp32 forward")


@pytest.mark.parametrize("shape", [(2, 3, 14, 28, 7), (1, 2, 28, 28, 14), (2, 1, 6, 9, 3)])
def test_fp32_forward_backward(shape):
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 3, torch.float32)
    dy = gen((B, C, H, W), 4, torch.float32)
    T = gen((C, (2 * w - 1) ** 2), 5, torch.float32, 0.02)
    xr, gr, Tr = to_np(x), to_np(dy), to_np(T)
    y = run_forward(x, T, w)
    check_f32(to_np(y), oracle.forward(xr, Tr, w), oracle.forward(np.abs(xr), np.abs(Tr), w), "y")
    dX, dT = wb.backward(x, T, dy, w)
    torch.cuda.synchronize()
    check_f32(to_np(dX), oracle.backward_dx(gr, Tr, w),
              oracle.backward_dx(np.abs(gr), np.abs(Tr), w), "dX")
    absdt = oracle.backward_dt(np.abs(xr), np.abs(gr), w)
    check_f32(to_np(dT), oracle.backward_dt(xr, gr, w), absdt, "dT")


@pytest.mark.parametrize("shape", BF16_SHAPES[:6], ids=lambda s: "x".join(map(str, s)))
def test_backward_bf16_small(shape):
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 6)
    dy = gen((B, C, H, W), 7)
    T = gen((C, (2 * w - 1) ** 2), 8, scale=0.02)
    dX, dT = wb.backward(x, T, dy, w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    assert wb.wbmm_last_path() == 1
    xr, gr, Tr = to_np(x), to_np(dy), to_np(T)
    check_bf16(to_np(dX), oracle.backward_dx(gr, Tr, w),
               forward_rowbound(gr, Tr[:, ::-1].copy(), w), "dX")
    check_bf16(to_np(dT), oracle.backward_dt(xr, gr, w), dt_bound(xr, gr, w), "dT")


# CUDA-core table gradient as G = dY X^T and diagonal sums (4 <= w <= 14):
# several tiles per channel with a ragged last tile, channels spread over
# several blocks and blocks whose tile range crosses channel boundaries
# (more tiles than the 148 blocks), a tile one window short of 64 (nw = 7),
# one band per tile (nw = 64) and the bf16 inputs that take this path (rows
# not 16-byte multiples), against the oracle.
DTG_SHAPES = [(35, 2, 28, 28, 14, torch.float32), (3, 2, 56, 49, 7, torch.float32),
              (20, 2, 30, 50, 10, torch.float32), (2, 2, 18, 576, 9, torch.float32),
              (30, 2, 10, 15, 5, torch.bfloat16), (5, 3, 8, 8, 4, torch.float32),
              (40, 60, 28, 28, 14, torch.float32), (4, 100, 56, 49, 7, torch.float32),
              (30, 40, 10, 15, 5, torch.bfloat16)]


@pytest.mark.parametrize("shape", DTG_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + str(s[5])[-4:])
def test_cuda_core_table_gradient(shape):
    B, C, H, W, w, dtype = shape
    x = gen((B, C, H, W), 60, dtype)
    dy = gen((B, C, H, W), 61, dtype)
    T = gen((C, (2 * w - 1) ** 2), 62, dtype, 0.02)
    dX, dT = wb.backward(x, T, dy, w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    xr, gr = to_np(x), to_np(dy)
    if dtype == torch.bfloat16:
        check_bf16(to_np(dT), oracle.backward_dt(xr, gr, w), dt_bound(xr, gr, w), "dT")
    else:
        check_f32(to_np(dT), oracle.backward_dt(xr, gr, w),
                  oracle.backward_dt(np.abs(xr), np.abs(gr), w), "dT")
    # the fixed summation order gives the same bits on every call
    dX2, dT2 = wb.backward(x, T, dy, w)
    torch.cuda.synchronize()
    assert torch.equal(dT, dT2)


def test_dt_is_deterministic():
    B, C, H, W, w = 9, 3, 56, 56, 14
    x, dy = gen((B, C, H, W), 9), gen((B, C, H, W), 10)
    T = gen((C, 729), 11, scale=0.02)
    runs = []
    for _ in range(4):
        _, dT = wb.backward(x, T, dy, w, need_dx=False)
        runs.append(dT.clone())
    torch.cuda.synchronize()
    for r in runs[1:]:
        assert torch.equal(r, runs[0])


def test_backward_both_gradients_share_the_device():
    # enough table-gradient tiles (40 channels x 16) for the two gradient
    # kernels to run side by side on disjoint SMs: dX equals the dX-only
    # call bit for bit (windows are independent of the grid), dT is
    # deterministic and within tolerance of the dT-only call (another grid,
    # so another fixed summation order)
    B, C, H, W, w = 64, 40, 56, 56, 14
    x, dy = gen((B, C, H, W), 30), gen((B, C, H, W), 31)
    T = gen((C, 729), 32, scale=0.02)
    dX1, _ = wb.backward(x, T, dy, w, need_dt=False)
    _, dT1 = wb.backward(x, T, dy, w, need_dx=False)
    runs = [wb.backward(x, T, dy, w) for _ in range(3)]
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    for dX, dT in runs:
        assert torch.equal(dX, dX1)
        assert torch.equal(dT, runs[0][1])
    xr, gr = to_np(x[:, :4]), to_np(dy[:, :4])
    check_bf16(to_np(runs[0][1][:4]), oracle.backward_dt(xr, gr, w), dt_bound(xr, gr, w),
               "dT with dX")
    check_bf16(to_np(runs[0][1]), to_np(dT1), dt_bound(to_np(x), to_np(dy), w), "dT vs dT-only")


# Degenerate and boundary window sizes: w = 1 (each channel a scalar gain,
# CUDA-core path), one window per image (tensor-core path, nh = nw = 1),
# w = 32 (largest register-tiled CUDA-core size) and w = 40 (plain CUDA-core
# kernel), forward and both gradients against the oracle.
EDGE_SHAPES = [(2, 3, 5, 7, 1, torch.bfloat16), (2, 3, 5, 7, 1, torch.float32),
               (3, 2, 14, 14, 14, torch.bfloat16), (1, 2, 64, 32, 32, torch.bfloat16),
               (1, 2, 40, 40, 40, torch.float32)]


@pytest.mark.parametrize("shape", EDGE_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + str(s[5])[-4:])
def test_edge_window_sizes(shape):
    B, C, H, W, w, dtype = shape
    x = gen((B, C, H, W), 40, dtype)
    dy = gen((B, C, H, W), 41, dtype)
    T = gen((C, (2 * w - 1) ** 2), 42, dtype, 0.02)
    y = run_forward(x, T, w)
    dX, dT = wb.backward(x, T, dy, w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    xr, gr, Tr = to_np(x), to_np(dy), to_np(T)
    if dtype == torch.bfloat16:
        check_bf16(to_np(y), oracle.forward(xr, Tr, w), forward_rowbound(xr, Tr, w), "y")
        check_bf16(to_np(dX), oracle.backward_dx(gr, Tr, w),
                   forward_rowbound(gr, Tr[:, ::-1].copy(), w), "dX")
        check_bf16(to_np(dT), oracle.backward_dt(xr, gr, w), dt_bound(xr, gr, w), "dT")
    else:
        check_f32(to_np(y), oracle.forward(xr, Tr, w),
                  oracle.forward(np.abs(xr), np.abs(Tr), w), "y")
        check_f32(to_np(dX), oracle.backward_dx(gr, Tr, w),
                  oracle.backward_dx(np.abs(gr), np.abs(Tr), w), "dX")
        check_f32(to_np(dT), oracle.backward_dt(xr, gr, w),
                  oracle.backward_dt(np.abs(xr), np.abs(gr), w), "dT")
    if w == 1:
        # one-position windows: y = T_c * x exactly (one product, rounded once)
        exp = (x.float() * T.float()[:, 0].view(1, C, 1, 1)).to(dtype)
        assert torch.equal(y, exp)


def test_unsupported_and_empty_shapes_launch_nothing():
    x = gen((1, 1, 65, 65), 43)
    T = gen((1, 129 * 129), 44, scale=0.02)
    y = torch.empty_like(x)
    before = wb.wbmm_launch_count()
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_forward(x, T, y, 65)                   # w above the supported maximum
    assert e.value.status == 5
    with pytest.raises(wb.WbmmError) as e:             # an empty batch is rejected
        wb._check(wb._lib.wbmm_forward(wb._p(x), wb._p(T), wb._p(y), 0, 1, 65, 65, 65, 1,
                                       wb._stream(None)))
    assert e.value.status == 1
    assert wb.wbmm_launch_count() == before


def test_full_size_fp32_forward_sampled():
    wl = synth.WORKLOADS["fwd_f32"]
    d = synth.draw(wl, seed=0)
    x, T = d["x"].to(DEV), d["T"].to(DEV)
    y = run_forward(x, T, wl.w)
    assert wb.wbmm_last_path() == 2
    bs, cs = sample_planes(wl.B, wl.C)
    xs, Ts = to_np(d["x"][bs][:, cs]), to_np(d["T"][cs])
    check_f32(to_np(y[bs][:, cs]), oracle.forward(xs, Ts, wl.w),
              oracle.forward(np.abs(xs), np.abs(Ts), wl.w), "fp32 forward")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_cache_matrices_bit_exact(dtype):
    for w in (3, 7, 14):
        T = gen((5, (2 * w - 1) ** 2), 12, dtype)
        M = wb.cache_matrices(T, w)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(M), oracle.expand(to_np(T), w))


@pytest.mark.parametrize("shape", [(3, 2, 56, 56, 14), (2, 3, 112, 56, 7), (2, 2, 48, 48, 16)])
def test_forward_cached_bf16(shape):
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 13)
    T = gen((C, (2 * w - 1) ** 2), 14, scale=0.02)
    M = wb.cache_matrices(T, w)
    y = wb.forward_cached(x, M, w)
    torch.cuda.synchronize()
    assert wb.wbmm_last_path() == 1
    xr, Tr = to_np(x), to_np(T)
    check_bf16(to_np(y), oracle.forward(xr, Tr, w), forward_rowbound(xr, Tr, w), "cached")
    # and the table path gives the identical bits
    assert torch.equal(y, wb.forward(x, T, w))
    # any matrix, not only a Toeplitz one
    Mr = gen((C, w * w, w * w), 15, scale=0.05)
    y2 = wb.forward_cached(x, Mr, w)
    torch.cuda.synchronize()
    Mn = to_np(Mr)
    ref = oracle.forward_cached(xr, Mn, w)
    rn = np.sqrt((Mn ** 2).sum(axis=2)).reshape(C, w, w)
    bound = window_norms(xr, w) * np.tile(rn, (1, H // w, W // w))[None]
    check_bf16(to_np(y2), ref, bound, "cached random M")


@pytest.mark.parametrize("dtype,w,k", [(torch.bfloat16, 14, 7), (torch.float32, 14, 7),
                                       (torch.bfloat16, 12, 4), (torch.float32, 6, 3)])
def test_reparam_merge(dtype, w, k):
    C = 3
    Tw = gen((C, (2 * w - 1) ** 2), 30, dtype, 0.02)
    Tk = gen((C, (2 * k - 1) ** 2), 31, dtype, 0.02)
    M = wb.reparam_merge(Tw, Tk, w, k)
    torch.cuda.synchronize()
    ref = oracle.reparam_merge(to_np(Tw), to_np(Tk), w, k)
    # the sum of two stored values is exact in fp32 here, so both sides round
    # it once to the storage type
    exp = torch.from_numpy(ref).to(torch.float32).to(dtype).to(DEV)
    assert torch.equal(M, exp)
    # the merged matrix computes the two branches: w-window plus k-window WBMM
    x = gen((2, C, 2 * w, 2 * w), 32, dtype)
    y = wb.forward_cached(x, M, w)
    torch.cuda.synchronize()
    xr = to_np(x)
    ref_y = oracle.forward(xr, to_np(Tw), w) + oracle.forward(xr, to_np(Tk), k)
    Mn = to_np(M)
    rn = np.sqrt((Mn ** 2).sum(axis=2)).reshape(C, w, w)
    bound = window_norms(xr, w) * np.tile(rn, (1, 2, 2))[None]
    if dtype == torch.bfloat16:
        check_bf16(to_np(y), ref_y, bound, "reparam forward")
    else:
        absref = oracle.forward_cached(np.abs(xr), np.abs(Mn), w)
        check_f32(to_np(y), ref_y, absref, "reparam forward")


def test_reparam_merge_argument_errors():
    Tw = gen((2, 27 * 27), 33, scale=0.02)
    Tk = gen((2, 9 * 9), 34, scale=0.02)
    M = torch.empty((2, 196, 196), dtype=torch.bfloat16, device=DEV)
    before = wb.wbmm_launch_count()
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_reparam_merge(Tw, Tk, M, 14, 5)       # 5 does not divide 14
    assert e.value.status == 1
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_reparam_merge(Tw, Tk, M, 14, 7)       # a 9x9 table where 7 needs 13x13
    assert e.value.status == 1
    Tk7 = gen((2, 13 * 13), 35, scale=0.02)
    alias = M.view(-1)[:2 * 27 * 27].view(2, 27 * 27)
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_reparam_merge(alias, Tk7, M, 14, 7)   # output overlaps a table
    assert e.value.status == 1
    assert wb.wbmm_launch_count() == before


# (B, C, H, W, w): tiles holding several whole planes (56x56, 42x56 with the
# tile cut to 30 bands, 70x112 with 15 and a partial last tile), planes of
# two tiles (224x224, 168x168 with tiles cut to 6 bands) and of three
# (336x224), one plane per tile (112x56 at w = 7), and w = 16 (the older
# fused kernel)
FUSED_SHAPES = [(3, 2, 56, 56, 14), (2, 3, 112, 56, 7), (2, 2, 48, 48, 16), (2, 3, 224, 224, 14),
                (2, 2, 42, 56, 14), (2, 2, 168, 168, 14), (1, 2, 336, 224, 14), (4, 2, 70, 112, 14)]


@pytest.mark.parametrize("shape", FUSED_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fused_cached_dw3x3_matches_two_calls(shape):
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 21)
    T = gen((C, (2 * w - 1) ** 2), 22, scale=0.02)
    K = gen((C, 1, 3, 3), 23, scale=1.0 / 3.0)
    M = wb.cache_matrices(T, w)
    z = wb.forward_cached(x, M, w, dw=K)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    assert wb.wbmm_last_path() == 1
    y = wb.forward_cached(x, M, w)
    z2 = wb.dw3x3(y, K)
    torch.cuda.synchronize()
    # y rounded to bf16 between the stages in both paths: the same bits
    assert torch.equal(z, z2)
    if H * W >= 224 * 224:
        # and within tolerance of the oracle's 3x3 of the oracle's y
        yr, Kr = to_np(y), to_np(K)
        ref = oracle.dw3x3(oracle.forward(to_np(x), to_np(T), w), Kr)
        bound = oracle.dw3x3(forward_rowbound(to_np(x), to_np(T), w), np.abs(Kr))
        check_bf16(to_np(z), ref, bound, "fused cached + 3x3")


def test_fused_cached_dw3x3_unsupported_shapes():
    # image rows that are not whole 16-byte vectors (W = 12)
    x = gen((2, 2, 12, 12), 24)
    M = wb.cache_matrices(gen((2, 49), 25, scale=0.02), 4)
    K = gen((2, 1, 3, 3), 26)
    before = wb.wbmm_launch_count()
    with pytest.raises(wb.WbmmError) as e:
        wb.forward_cached(x, M, 4, dw=K)
    assert e.value.status == 5
    # fp32 maps
    xf = gen((1, 2, 14, 14), 27, torch.float32)
    Mf = wb.cache_matrices(gen((2, 169), 28, torch.float32, 0.02), 7)
    with pytest.raises(wb.WbmmError) as e:
        wb.forward_cached(xf, Mf, 7, dw=gen((2, 1, 3, 3), 29, torch.float32))
    assert e.value.status == 5
    assert wb.wbmm_launch_count() == before + 1     # only the fp32 cache_matrices


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
# scalar path (W % 8 != 0) and the 16-byte-vector path: one vector per row,
# one 32-vector chunk, several chunks with a ragged last one, a single row
@pytest.mark.parametrize("hw", [(37, 70), (40, 64), (33, 8), (19, 264), (9, 520), (1, 16)])
def test_dw3x3(dtype, hw):
    y = gen((3, 4) + hw, 16, dtype)
    K = gen((4, 1, 3, 3), 17, dtype, 1.0 / 3.0)
    z = wb.dw3x3(y, K)
    torch.cuda.synchronize()
    yr, Kr = to_np(y), to_np(K)
    ref = oracle.dw3x3(yr, Kr)
    if dtype == torch.float32:
        absdot = oracle.dw3x3(np.abs(yr), np.abs(Kr))
        check_f32(to_np(z), ref, absdot, "dw3x3 fp32")
    else:
        bound = oracle.dw3x3(np.abs(yr), np.abs(Kr))
        check_bf16(to_np(z), ref, bound, "dw3x3 bf16")


def test_guard_bands_untouched():
    B, C, H, W, w = 9, 3, 56, 56, 14
    n = B * C * H * W
    pad = 4096
    x = gen((B, C, H, W), 18)
    T = gen((C, 729), 19, scale=0.02)
    buf = torch.full((n + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    y = buf[pad:pad + n].view(B, C, H, W)
    wb.wbmm_forward(x, T, y, w)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 7.0) and torch.all(buf[pad + n:] == 7.0)
    assert torch.equal(y, wb.forward(x, T, w))


def test_argument_errors_launch_nothing():
    x = gen((1, 2, 28, 28), 20)
    T = gen((2, 729), 21, scale=0.02)
    y = torch.empty_like(x)
    before = wb.wbmm_launch_count()
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_forward(x, T, y, 5)                    # 28 % 5 != 0
    assert e.value.status == 2
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_forward(x, T, x, 14)                   # output overlaps input
    assert e.value.status == 1
    big = torch.empty(x.numel() + 8, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_forward(x, T, big[1:1 + x.numel()].view_as(x), 14)  # 2-byte offset
    assert e.value.status == 4
    dT = torch.empty((2, 729), dtype=torch.float32, device=DEV)
    ws = torch.empty(4, dtype=torch.float32, device=DEV)
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_backward(x, T, x, None, dT, ws, 14)    # workspace too small
    assert e.value.status == 6
    assert wb.wbmm_launch_count() == before


def test_bounded_wait_reports_timeout_and_context_survives():
    wb.wbmm_wait_selftest(2_000_000)
    assert wb.wbmm_get_device_status() == 8
    assert wb.wbmm_get_device_status() == 0          # cleared
    x = gen((2, 2, 28, 28), 22)
    T = gen((2, 729), 23, scale=0.02)
    y = run_forward(x, T, 14)
    ref = oracle.forward(to_np(x), to_np(T), 14)
    check_bf16(to_np(y), ref, forward_rowbound(to_np(x), to_np(T), 14), "after timeout")


# ---------------------------------------------------------------- full size

def sample_planes(B, C, nb=3, nc=3, seed=0):
    g = np.random.default_rng(seed)
    bs = sorted(set([0, B - 1] + list(g.integers(0, B, nb))))
    cs = sorted(set([0, C - 1] + list(g.integers(0, C, nc))))
    return bs, cs


@pytest.mark.parametrize("name", ["fwd_bf16", "sweep_w7", "sweep_w14", "sweep_w28"])
def test_full_size_forward_sampled(name):
    wl = synth.WORKLOADS[name]
    d = synth.draw(wl, seed=0)
    x, T = d["x"].to(DEV), d["T"].to(DEV)
    y = run_forward(x, T, wl.w)
    bs, cs = sample_planes(wl.B, wl.C)
    xs = to_np(d["x"][bs][:, cs])
    Ts = to_np(d["T"][cs])
    ref = oracle.forward(xs, Ts, wl.w)
    got = to_np(y[bs][:, cs])
    check_bf16(got, ref, forward_rowbound(xs, Ts, wl.w), name)


def test_full_size_training_step_sampled():
    wl = synth.WORKLOADS["train_bf16"]
    d = synth.draw(wl, seed=0)
    x, T, dy = d["x"].to(DEV), d["T"].to(DEV), d["dY"].to(DEV)
    y = run_forward(x, T, wl.w)
    dX, dT = wb.backward(x, T, dy, wl.w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    bs, cs = sample_planes(wl.B, wl.C)
    xs, gs, Ts = to_np(d["x"][bs][:, cs]), to_np(d["dY"][bs][:, cs]), to_np(d["T"][cs])
    check_bf16(to_np(y[bs][:, cs]), oracle.forward(xs, Ts, wl.w),
               forward_rowbound(xs, Ts, wl.w), "train y")
    check_bf16(to_np(dX[bs][:, cs]), oracle.backward_dx(gs, Ts, wl.w),
               forward_rowbound(gs, Ts[:, ::-1].copy(), wl.w), "train dX")
    # dT of a channel sums over every image: the oracle takes whole channels
    xc, gc = to_np(d["x"][:, cs]), to_np(d["dY"][:, cs])
    check_bf16(to_np(dT[cs]), oracle.backward_dt(xc, gc, wl.w), dt_bound(xc, gc, wl.w),
               "train dT")


def test_full_size_cached_dw_sampled():
    wl = synth.WORKLOADS["hires_cached_dw"]
    d = synth.draw(wl, seed=0)
    x, T, K = d["x"].to(DEV), d["T"].to(DEV), d["K"].to(DEV)
    M = wb.cache_matrices(T, wl.w)
    y = wb.forward_cached(x, M, wl.w)
    z = wb.dw3x3(y, K)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    bs, cs = sample_planes(wl.B, wl.C)
    xs, Ts, Ks = to_np(d["x"][bs][:, cs]), to_np(d["T"][cs]), to_np(d["K"][cs])
    yref = oracle.forward(xs, Ts, wl.w)
    check_bf16(to_np(y[bs][:, cs]), yref, forward_rowbound(xs, Ts, wl.w), "hires y")
    zref = oracle.dw3x3(yref, Ks)
    # |z - zref| <= sum |K| * (|y - yref| + rounding of z): bound by the 3x3 of
    # the forward row bound
    zb = oracle.dw3x3(forward_rowbound(xs, Ts, wl.w), np.abs(Ks))
    check_bf16(to_np(z[bs][:, cs]), zref, zb, "hires z")
    # the fused launch gives the two calls' bits at full size
    zf = wb.forward_cached(x, M, wl.w, dw=K)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    assert torch.equal(zf, z)


def test_full_size_fp32_training_step_sampled():
    # the fp32 path (CUDA cores) on the training workload, as bench.py
    # --workload train32 runs it: sampled planes for y and dX, whole sampled
    # channels for dT
    wl = synth.WORKLOADS["train_f32"]
    d = synth.draw(wl, seed=0)
    x, T, dy = d["x"].to(DEV), d["T"].to(DEV), d["dY"].to(DEV)
    y = run_forward(x, T, wl.w)
    dX, dT = wb.backward(x, T, dy, wl.w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    assert wb.wbmm_last_path() == 2
    bs, cs = sample_planes(wl.B, wl.C)
    xs, gs, Ts = to_np(d["x"][bs][:, cs]), to_np(d["dY"][bs][:, cs]), to_np(d["T"][cs])
    check_f32(to_np(y[bs][:, cs]), oracle.forward(xs, Ts, wl.w),
              oracle.forward(np.abs(xs), np.abs(Ts), wl.w), "train32 y")
    check_f32(to_np(dX[bs][:, cs]), oracle.backward_dx(gs, Ts, wl.w),
              oracle.backward_dx(np.abs(gs), np.abs(Ts), wl.w), "train32 dX")
    xc, gc = to_np(d["x"][:, cs]), to_np(d["dY"][:, cs])
    check_f32(to_np(dT[cs]), oracle.backward_dt(xc, gc, wl.w),
              oracle.backward_dt(np.abs(xc), np.abs(gc), wl.w), "train32 dT")


def test_full_size_fp32_cached_dw_sampled():
    wl = synth.WORKLOADS["hires_cached_dw_f32"]
    d = synth.draw(wl, seed=0)
    x, T, K = d["x"].to(DEV), d["T"].to(DEV), d["K"].to(DEV)
    M = wb.cache_matrices(T, wl.w)
    y = wb.forward_cached(x, M, wl.w)
    z = wb.dw3x3(y, K)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    bs, cs = sample_planes(wl.B, wl.C)
    xs, Ts, Ks = to_np(d["x"][bs][:, cs]), to_np(d["T"][cs]), to_np(d["K"][cs])
    yref = oracle.forward(xs, Ts, wl.w)
    yabs = oracle.forward(np.abs(xs), np.abs(Ts), wl.w)
    check_f32(to_np(y[bs][:, cs]), yref, yabs, "cached32 y")
    # the 3x3 of the GPU's own y: z's error against that is the stencil's
    # fp32 accumulation alone
    yg = to_np(y[bs][:, cs])
    check_f32(to_np(z[bs][:, cs]), oracle.dw3x3(yg, Ks), oracle.dw3x3(np.abs(yg), np.abs(Ks)),
              "cached32 z")


def test_full_size_reparam_sampled():
    # the high-resolution shape through one matrix merged from a 14x14 and a
    # 7x7 table, as bench.py --workload reparam runs it
    wl = synth.WORKLOADS["hires_reparam"]
    k = synth.REPARAM_SMALL_WINDOW
    d = synth.draw(wl, seed=0)
    x, T, Tk = d["x"].to(DEV), d["T"].to(DEV), d["Tk"].to(DEV)
    M = wb.reparam_merge(T, Tk, wl.w, k)
    y = wb.forward_cached(x, M, wl.w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    bs, cs = sample_planes(wl.B, wl.C)
    xs = to_np(d["x"][bs][:, cs])
    ref = oracle.forward(xs, to_np(d["T"][cs]), wl.w) + oracle.forward(xs, to_np(d["Tk"][cs]), k)
    Mn = to_np(M[cs])
    rn = np.sqrt((Mn ** 2).sum(axis=2)).reshape(len(cs), wl.w, wl.w)
    bound = window_norms(xs, wl.w) * np.tile(rn, (1, wl.H // wl.w, wl.W // wl.w))[None]
    check_bf16(to_np(y[bs][:, cs]), ref, bound, "reparam y")


@pytest.mark.parametrize("shape", [(3, 2, 56, 56, 14), (2, 3, 35, 70, 7), (1, 2, 15, 45, 5),
                                   (5, 1, 42, 28, 14)], ids=lambda s: "x".join(map(str, s)))
def test_fp32_cached_forward_equals_table_forward(shape):
    # both CUDA-core kernels sum each output's d products in (r, s) order
    # with fused multiply-adds, and the cached matrix holds exact copies of
    # table entries: the results agree bit for bit; also checked against the
    # oracle (window counts that are not multiples of the 64-window tile)
    B, C, H, W, w = shape
    x = gen((B, C, H, W), 40, torch.float32)
    T = gen((C, (2 * w - 1) ** 2), 41, torch.float32, 0.02)
    M = wb.cache_matrices(T, w)
    yc = wb.forward_cached(x, M, w)
    yt = wb.forward(x, T, w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    assert torch.equal(yc, yt)
    xr, Tr = to_np(x), to_np(T)
    check_f32(to_np(yc), oracle.forward(xr, Tr, w), oracle.forward(np.abs(xr), np.abs(Tr), w),
              "fp32 cached")
