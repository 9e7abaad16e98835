"""GPU: the table gradient's hand-off between CTAs, through the C ABI.

A channel whose windows are split between CTAs is finished by the last CTA
to arrive at the channel's counter in the workspace; every launch leaves the
counters at zero.  These tests pin the properties that design promises:
consecutive calls on one workspace with different inputs, graph replays
with new inputs (the same launch parameters every time), partial tables left
over from an earlier call (poisoned with NaN here) never being read, and the
counters reading zero after every call.  Each result is compared with the
fp64 oracle.
"""
import numpy as np
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

# dT-only calls whose channels are split between CTAs: 9 images of 56x56 at
# w = 14 make 3 tiles per channel and a 9-CTA grid (3 CTAs per channel);
# 3 images of 40x40 at w = 5 make 3 tiles per channel and a 6-CTA grid
SPLIT_SHAPES = [(9, 3, 56, 56, 14), (3, 2, 40, 40, 5)]
# both gradients side by side (640 tiles: dX on 59 SMs, dT on the other 89):
# 40 channels over 89 CTAs, every channel split
BOTH_SHAPE = (64, 40, 56, 56, 14)


def gen(shape, seed, scale=1.0):
    return synth.draw_tensor(shape, seed, "f32", scale).to(torch.bfloat16).to(DEV)


def workspace(B, C, H, W, w):
    n = wb.wbmm_backward_workspace_bytes(B, C, H, W, w, torch.bfloat16) // 4
    return torch.zeros(n, dtype=torch.float32, device=DEV)


def counters(ws):
    """The workspace's counter region (one arrival counter per channel)."""
    return ws[:wb.WBMM_DT_COUNTER_WORDS].view(torch.int32)


def check_dt(dT, x, dy, w, what, channels=None):
    cs = list(range(x.shape[1])) if channels is None else channels
    xr, gr = to_np(x[:, cs]), to_np(dy[:, cs])
    check_bf16(to_np(dT[cs]), oracle.backward_dt(xr, gr, w), dt_bound(xr, gr, w), what)


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_consecutive_calls_share_a_workspace(shape):
    B, C, H, W, w = shape
    ws = workspace(B, C, H, W, w)
    dT = torch.empty((C, (2 * w - 1) ** 2), dtype=torch.float32, device=DEV)
    for call in range(3):
        x, dy = gen((B, C, H, W), 100 + 2 * call), gen((B, C, H, W), 101 + 2 * call)
        if call == 2:
            # partial tables left by the previous call must never be read
            ws[wb.WBMM_DT_COUNTER_WORDS:].fill_(float("nan"))
        wb.wbmm_backward(x, None, dy, None, dT, ws, w)
        torch.cuda.synchronize()
        assert wb.wbmm_get_device_status() == 0
        assert torch.all(counters(ws) == 0), "counters not reset"
        assert torch.isfinite(dT).all()
        check_dt(dT, x, dy, w, "dT, call %d" % call)


def test_one_workspace_serves_calls_of_different_shapes():
    # the counter words are the same for every shape: calls of other shapes
    # that wrote partial tables into the same buffer leave them zero
    n = max(wb.wbmm_backward_workspace_bytes(*s, torch.bfloat16) for s in SPLIT_SHAPES) // 4
    ws = torch.zeros(n, dtype=torch.float32, device=DEV)
    for rnd in range(2):
        for i, (B, C, H, W, w) in enumerate(SPLIT_SHAPES):
            x, dy = gen((B, C, H, W), 140 + 4 * rnd + 2 * i), gen((B, C, H, W), 141 + 4 * rnd + 2 * i)
            dT = torch.full((C, (2 * w - 1) ** 2), float("nan"), dtype=torch.float32, device=DEV)
            wb.wbmm_backward(x, None, dy, None, dT, ws, w)
            torch.cuda.synchronize()
            assert wb.wbmm_get_device_status() == 0
            assert torch.all(counters(ws) == 0), "counters not reset"
            check_dt(dT, x, dy, w, "shape %d, round %d" % (i, rnd))


@pytest.mark.parametrize("shape", SPLIT_SHAPES + [BOTH_SHAPE], ids=lambda s: "x".join(map(str, s)))
def test_graph_replay_with_new_inputs(shape):
    # a captured backward call replays with the same launch parameters every
    # time; each replay must see only its own partial tables
    B, C, H, W, w = shape
    both = shape == BOTH_SHAPE
    x = torch.empty((B, C, H, W), dtype=torch.bfloat16, device=DEV)
    dy = torch.empty_like(x)
    dX = torch.empty_like(x) if both else None
    T = gen((C, (2 * w - 1) ** 2), 120, scale=0.02)
    dT = torch.empty((C, (2 * w - 1) ** 2), dtype=torch.float32, device=DEV)
    ws = workspace(B, C, H, W, w)
    x.copy_(gen((B, C, H, W), 121))
    dy.copy_(gen((B, C, H, W), 122))
    wb.wbmm_backward(x, T, dy, dX, dT, ws, w)       # configures kernels before capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        wb.wbmm_backward(x, T, dy, dX, dT, ws, w)
    torch.cuda.synchronize()
    channels = [0, 1, C // 2, C - 1] if both else None
    for rep in range(3):
        x.copy_(gen((B, C, H, W), 130 + 2 * rep))
        dy.copy_(gen((B, C, H, W), 131 + 2 * rep))
        dT.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert wb.wbmm_get_device_status() == 0
        assert torch.all(counters(ws) == 0), "counters not reset"
        check_dt(dT, x, dy, w, "replay %d" % rep, channels)
        if both:
            xs, gs, Ts = to_np(x[:2, channels]), to_np(dy[:2, channels]), to_np(T[channels])
            check_bf16(to_np(dX[:2, channels]), oracle.backward_dx(gs, Ts, w),
                       forward_rowbound(gs, Ts[:, ::-1].copy(), w), "replay %d dX" % rep)
    del g
