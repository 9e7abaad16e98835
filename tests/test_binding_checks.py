"""The Python binding's buffer checks, without a GPU.

The C ABI takes plain pointers, so the binding checks what the library
cannot see: each buffer's device, dtype and element count against the call's
map.  CPU tensors stand in for device tensors here: a call whose buffers pass
the checks reaches the pointer conversion, which refuses non-CUDA tensors
with ValueError before anything is launched.  (The device check compares
CUDA device indices and needs two GPUs to fail.)
"""
import importlib.util
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wb():
    spec = importlib.util.spec_from_file_location(
        "_wbmm_build", os.path.join(ROOT, "windowed_matmul_conv_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    import windowed_matmul_conv_b200 as mod
    return mod


BF = torch.bfloat16


def maps(B=2, C=3, H=28, W=28, dtype=BF):
    return torch.zeros((B, C, H, W), dtype=dtype)


def status_of(fn, *a):
    import windowed_matmul_conv_b200 as mod
    try:
        fn(*a)
    except mod.WbmmError as e:
        return e.status
    except ValueError:
        return "passed"          # checks passed; only the CUDA pointer was refused
    raise AssertionError("no exception")


def test_forward_buffers(wb):
    x, T, y = maps(), torch.zeros((3, 729), dtype=BF), maps()
    assert status_of(wb.wbmm_forward, x, T, y, 14) == "passed"
    assert status_of(wb.wbmm_forward, x, T[:2], y, 14) == 1            # table too short
    assert status_of(wb.wbmm_forward, x, T, y[:1], 14) == 1            # output too short
    assert status_of(wb.wbmm_forward, x, T.float(), y, 14) == 3        # table dtype
    assert status_of(wb.wbmm_forward, x, T, y.float(), 14) == 3        # output dtype
    # a longer table than the window needs is fine (the library rejects the shape)
    assert status_of(wb.wbmm_forward, x, T, y, 7) == "passed"


def test_backward_buffers(wb):
    x, dY, dX = maps(), maps(), maps()
    T = torch.zeros((3, 729), dtype=BF)
    dT = torch.zeros((3, 729), dtype=torch.float32)
    ws = torch.zeros(16, dtype=torch.float32)
    assert status_of(wb.wbmm_backward, x, T, dY, dX, dT, ws, 14) == "passed"
    assert status_of(wb.wbmm_backward, None, T, dY, dX, None, None, 14) == "passed"
    assert status_of(wb.wbmm_backward, x, None, dY, None, dT, ws, 14) == "passed"
    assert status_of(wb.wbmm_backward, x[:1], T, dY, dX, dT, ws, 14) == 1
    assert status_of(wb.wbmm_backward, x, T, dY, dX[:1], dT, ws, 14) == 1
    assert status_of(wb.wbmm_backward, x, T, dY, dX, dT[:2], ws, 14) == 1
    assert status_of(wb.wbmm_backward, x, T, dY, dX, dT.to(BF), ws, 14) == 3   # dT is fp32
    assert status_of(wb.wbmm_backward, x.float(), T, dY, dX, dT, ws, 14) == 3
    assert status_of(wb.wbmm_backward_dt_static, x, dY, dT, 14) == "passed"
    assert status_of(wb.wbmm_backward_dt_static, x, dY, dT[:1], 14) == 1
    assert status_of(wb.wbmm_backward_dt_static, x[:1], dY, dT, 14) == 1


def test_cached_path_buffers(wb):
    T = torch.zeros((3, 729), dtype=BF)
    M = torch.zeros((3, 196, 196), dtype=BF)
    assert status_of(wb.wbmm_cache_matrices, T, M, 14) == "passed"
    assert status_of(wb.wbmm_cache_matrices, T, M[:2], 14) == 1
    assert status_of(wb.wbmm_cache_matrices, T[:, :169], M, 14) == 1
    Tk = torch.zeros((3, 169), dtype=BF)
    assert status_of(wb.wbmm_reparam_merge, T, Tk, M, 14, 7) == "passed"
    assert status_of(wb.wbmm_reparam_merge, T, Tk[:, :25], M, 14, 7) == 1
    assert status_of(wb.wbmm_reparam_merge, T, Tk.float(), M, 14, 7) == 3
    x, out = maps(), maps()
    K = torch.zeros((3, 1, 3, 3), dtype=BF)
    assert status_of(wb.wbmm_forward_cached, x, M, None, out, 14) == "passed"
    assert status_of(wb.wbmm_forward_cached, x, M, K, out, 14) == "passed"
    assert status_of(wb.wbmm_forward_cached, x, M[:1], K, out, 14) == 1
    assert status_of(wb.wbmm_forward_cached, x, M, K[:2], out, 14) == 1
    assert status_of(wb.wbmm_forward_cached, x, M, K, out[:, :2], 14) == 1
    assert status_of(wb.wbmm_dw3x3, x, K, out) == "passed"
    assert status_of(wb.wbmm_dw3x3, x, K.float(), out) == 3
    assert status_of(wb.wbmm_dw3x3, x, K, out[:1]) == 1


def test_workspace_size_dtypes(wb):
    assert wb.wbmm_backward_workspace_bytes(2, 3, 28, 28, 14, torch.float32) > 0
    with pytest.raises(TypeError):
        wb.wbmm_backward_workspace_bytes(2, 3, 28, 28, 14, torch.float16)
