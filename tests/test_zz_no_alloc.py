"""wbmm_backward_dt_static: the table gradient for callers that cannot allocate.

Hosts with a fixed device-memory budget, plugins inside frameworks that own
every device allocation, and paths where cudaMalloc would synchronise the
device cannot hand wbmm_backward a workspace.  This entry point keeps the
partial tables in a fixed array inside the library instead.  The test calls
it through the C ABI twice in a row per shape, with new inputs for the
second call, and checks each result against the fp64 oracle within the
bf16/fp32 tolerances of every parity test, and against wbmm_backward's dT
on the same inputs, which it must equal bit for bit (same kernels, same
partial split).
This file sorts last so a run that stops at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from parity_util import check_bf16, check_f32, dt_bound, to_np

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import windowed_matmul_conv_b200 as wb  # noqa: E402

# in this order, each shape's calls follow the previous shape's in the same
# array: a CUDA-core call between tensor-core calls must leave the arrival
# counters intact
SHAPES = [
    (9, 3, 56, 56, 14, torch.bfloat16),   # tensor-core path, several tiles
    (2, 3, 14, 28, 7, torch.float32),     # CUDA-core fp32 path
    (3, 2, 40, 40, 5, torch.bfloat16),    # odd window size, another shape
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + str(s[5])[-4:])
def test_static_scratch_matches_oracle_and_workspace_path(shape):
    B, C, H, W, w, dtype = shape
    for call in range(2):
        x = synth.draw_tensor((B, C, H, W), 41 + 2 * call, "f32").to(dtype).cuda()
        dy = synth.draw_tensor((B, C, H, W), 42 + 2 * call, "f32").to(dtype).cuda()
        dT = torch.full((C, (2 * w - 1) ** 2), float("nan"), dtype=torch.float32, device="cuda")
        wb.wbmm_backward_dt_static(x, dy, dT, w)
        torch.cuda.synchronize()
        assert wb.wbmm_get_device_status() == 0
        xr, gr = to_np(x), to_np(dy)
        ref = oracle.backward_dt(xr, gr, w)
        if dtype == torch.bfloat16:
            check_bf16(to_np(dT), ref, dt_bound(xr, gr, w), "static dT, call %d" % call)
        else:
            absdt = oracle.backward_dt(np.abs(xr), np.abs(gr), w)
            check_f32(to_np(dT), ref, absdt, "static dT, call %d" % call)
        _, ws_dT = wb.backward(x, None, dy, w, need_dx=False)
        torch.cuda.synchronize()
        assert torch.equal(dT, ws_dT)


def test_static_scratch_rejects_oversized_calls():
    # 2 images x 4096 channels of 56x56 at w=14 need 4096 x 729 partial
    # entries, more than the 2^20-float array holds: rejected before launch.
    x = torch.zeros((2, 4096, 56, 56), dtype=torch.bfloat16, device="cuda")
    dT = torch.empty((4096, 729), dtype=torch.float32, device="cuda")
    before = wb.wbmm_launch_count()
    with pytest.raises(wb.WbmmError) as e:
        wb.wbmm_backward_dt_static(x, x.clone(), dT, 14)
    assert e.value.status == 6
    assert wb.wbmm_launch_count() == before
