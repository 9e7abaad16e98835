"""GPU: the tensor-core pipelines' failure handling and their independence of
the load ring's depth, through the C ABI.

A bounded wait that runs out inside a production kernel is provoked on the
host side (wbmm_debug_set: the load producer of CTA 0 skips one tile, so the
transform's wait for that tile never completes) under a short wait budget.
The kernel must give up, drain its copies and MMAs, release its tensor
memory and return; the status word reports WBMM_ERR_TIMEOUT, and the next
normal call on the same context matches the fp64 oracle.  Nothing here faults
or hangs a GPU: every wait in these kernels is bounded.

Race detection by construction: the same calls with the load ring capped at
its minimum depth (2 slots) and at its default depth give bit-identical
outputs.
"""
import pytest
import torch

import oracle
import synth
from parity_util import check_bf16, dt_bound, forward_rowbound, to_np

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import windowed_matmul_conv_b200 as wb  # noqa: E402

DEV = "cuda:0"
SHORT_BUDGET = 20_000_000     # SM cycles, ~10 ms at 2 GHz


def gen(shape, seed, scale=1.0):
    return synth.draw_tensor(shape, seed, "f32", scale).to(torch.bfloat16).to(DEV)


@pytest.fixture
def short_waits():
    wb.wbmm_set_wait_budget(SHORT_BUDGET)
    try:
        yield
    finally:
        wb.wbmm_set_wait_budget(0)
        wb.wbmm_debug_set(wb.WBMM_DEBUG_SKIP_LOAD_WINDOW_MAJOR, -1)
        wb.wbmm_debug_set(wb.WBMM_DEBUG_SKIP_LOAD_TABLE_GRAD, -1)
        wb.wbmm_get_device_status()


def test_window_major_kernel_abort_path(short_waits):
    B, C, H, W, w = 4, 6, 56, 56, 14
    x, T = gen((B, C, H, W), 201), gen((C, 729), 202, scale=0.02)
    assert wb.wbmm_get_device_status() == 0
    wb.wbmm_debug_set(wb.WBMM_DEBUG_SKIP_LOAD_WINDOW_MAJOR, 0)
    wb.forward(x, T, w)
    assert wb.wbmm_last_path() == 1
    assert wb.wbmm_get_device_status() == 8, "the skipped load must end in a timeout"
    assert wb.wbmm_get_device_status() == 0, "status is cleared once read"
    wb.wbmm_set_wait_budget(0)
    # the context survives: the next calls are correct
    y = wb.forward(x, T, w)
    dX, _ = wb.backward(None, T, x, w, need_dt=False)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    xr, Tr = to_np(x), to_np(T)
    check_bf16(to_np(y), oracle.forward(xr, Tr, w), forward_rowbound(xr, Tr, w), "y after abort")
    check_bf16(to_np(dX), oracle.backward_dx(xr, Tr, w),
               forward_rowbound(xr, Tr[:, ::-1].copy(), w), "dX after abort")


def test_table_gradient_kernel_abort_path(short_waits):
    # 9 images of 56x56: channels split between CTAs, so the aborted launch
    # also exercises the arrival counters, which must be zero again after it
    B, C, H, W, w = 9, 3, 56, 56, 14
    x, dy = gen((B, C, H, W), 211), gen((B, C, H, W), 212)
    n = wb.wbmm_backward_workspace_bytes(B, C, H, W, w, torch.bfloat16) // 4
    ws = torch.zeros(n, dtype=torch.float32, device=DEV)
    dT = torch.empty((C, 729), dtype=torch.float32, device=DEV)
    wb.wbmm_debug_set(wb.WBMM_DEBUG_SKIP_LOAD_TABLE_GRAD, 0)
    wb.wbmm_backward(x, None, dy, None, dT, ws, w)
    assert wb.wbmm_get_device_status() == 8, "the skipped load must end in a timeout"
    assert torch.all(ws[:wb.WBMM_DT_COUNTER_WORDS].view(torch.int32) == 0)
    wb.wbmm_set_wait_budget(0)
    wb.wbmm_backward(x, None, dy, None, dT, ws, w)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0
    xr, gr = to_np(x), to_np(dy)
    check_bf16(to_np(dT), oracle.backward_dt(xr, gr, w), dt_bound(xr, gr, w), "dT after abort")


@pytest.mark.parametrize("shape", [(9, 3, 56, 56, 14), (6, 3, 40, 40, 5), (64, 40, 56, 56, 14)],
                         ids=lambda s: "x".join(map(str, s)))
def test_ring_depth_does_not_change_results(shape):
    B, C, H, W, w = shape
    x, dy = gen((B, C, H, W), 221), gen((B, C, H, W), 222)
    T = gen((C, (2 * w - 1) ** 2), 223, scale=0.02)

    def run():
        y = wb.forward(x, T, w)
        dX, dT = wb.backward(x, T, dy, w)
        dX1, _ = wb.backward(x, T, dy, w, need_dt=False)
        _, dT1 = wb.backward(x, T, dy, w, need_dx=False)
        torch.cuda.synchronize()
        assert wb.wbmm_get_device_status() == 0
        return [y, dX, dT, dX1, dT1]

    ref = run()
    try:
        wb.wbmm_debug_set(wb.WBMM_DEBUG_RING_CAP, 2)
        got = run()
    finally:
        wb.wbmm_debug_set(wb.WBMM_DEBUG_RING_CAP, 0)
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
