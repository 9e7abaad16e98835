"""Randomised properties of the WBMM oracle (hypothesis, small shapes).

The fixed-shape pins in test_oracle_pins.py tie each oracle function to a
library routine, a closed form or an exact special case; these properties
draw the window size, the map shape and the values at random and check
structure the operator has by its definition: linearity in x and in T, the
adjoint identities of both gradients, equivariance under a shift by whole
windows, the per-window depthwise-convolution equivalence for any odd
kernel no wider than the window, the 3x3 mixing against torch, and the
reparameterisation merge against the sum of its two branches.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import Oracle

SETTINGS = settings(max_examples=20, deadline=None,
                    suppress_health_check=[HealthCheck.function_scoped_fixture])


@st.composite
def problems(draw, wmax=6):
    w = draw(st.integers(1, wmax))
    B = draw(st.integers(1, 3))
    C = draw(st.integers(1, 3))
    nh = draw(st.integers(1, 3))
    nw = draw(st.integers(1, 3))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return w, (B, C, nh * w, nw * w), seed


def arrays(seed, *shapes):
    g = np.random.default_rng(seed)
    return [g.standard_normal(s) for s in shapes]


def close(a, b, tol=1e-12):
    scale = max(1.0, float(np.abs(a).max(initial=0.0)), float(np.abs(b).max(initial=0.0)))
    return float(np.abs(a - b).max(initial=0.0)) <= tol * scale


@SETTINGS
@given(problems())
def test_linear_in_input_and_table(oracle_mod, prob):
    orc = oracle_mod.default()
    w, shp, seed = prob
    t = (shp[1], (2 * w - 1) ** 2)
    x1, x2, T1, T2 = arrays(seed, shp, shp, t, t)
    a, b = 0.75, -1.5
    assert close(orc.forward(a * x1 + b * x2, T1, w),
                 a * orc.forward(x1, T1, w) + b * orc.forward(x2, T1, w))
    assert close(orc.forward(x1, a * T1 + b * T2, w),
                 a * orc.forward(x1, T1, w) + b * orc.forward(x1, T2, w))


@SETTINGS
@given(problems())
def test_gradients_are_adjoints(oracle_mod, prob):
    orc = oracle_mod.default()
    w, shp, seed = prob
    t = (shp[1], (2 * w - 1) ** 2)
    x, dy, T = arrays(seed, shp, shp, t)
    lhs = float(np.sum(dy * orc.forward(x, T, w)))
    assert abs(lhs - float(np.sum(orc.backward_dx(dy, T, w) * x))) <= 1e-11 * max(1.0, abs(lhs))
    assert abs(lhs - float(np.sum(orc.backward_dt(x, dy, w) * T))) <= 1e-11 * max(1.0, abs(lhs))


@SETTINGS
@given(problems(), st.integers(0, 2), st.integers(0, 2))
def test_shift_by_whole_windows(oracle_mod, prob, di, dj):
    # rolling the map by whole windows rolls the output the same way
    orc = oracle_mod.default()
    w, shp, seed = prob
    x, T = arrays(seed, shp, (shp[1], (2 * w - 1) ** 2))
    sh = (di * w, dj * w)
    assert np.array_equal(orc.forward(np.roll(x, sh, axis=(2, 3)), T, w),
                          np.roll(orc.forward(x, T, w), sh, axis=(2, 3)))


@SETTINGS
@given(problems(wmax=7), st.integers(0, 3))
def test_window_depthwise_convolution(oracle_mod, prob, kh):
    # a table supported on |offset| <= k//2 is a k x k cross-correlation
    # applied to each window as its own zero-padded image
    orc = oracle_mod.default()
    w, (B, C, H, W), seed = prob
    k = min(2 * kh + 1, 2 * ((w - 1) // 2) + 1)
    (K,) = arrays(seed, (C, k, k))
    T = np.zeros((C, (2 * w - 1) ** 2))
    h = k // 2
    for a in range(k):
        for e in range(k):
            T[:, (w - 1 + h - a) * (2 * w - 1) + (w - 1 + h - e)] = K[:, a, e]
    (x,) = arrays(seed + 1, (B, C, H, W))
    nh, nw = H // w, W // w
    xw = x.reshape(B, C, nh, w, nw, w).transpose(0, 2, 4, 1, 3, 5).reshape(-1, C, w, w)
    ref = F.conv2d(torch.from_numpy(xw), torch.from_numpy(K).unsqueeze(1), padding=h,
                   groups=C).numpy()
    ref = ref.reshape(B, nh, nw, C, w, w).transpose(0, 3, 1, 4, 2, 5).reshape(B, C, H, W)
    assert close(orc.forward(x, T, w), ref)


@SETTINGS
@given(st.integers(1, 2), st.integers(1, 4), st.integers(1, 9), st.integers(1, 9),
       st.integers(0, 2 ** 31 - 1))
def test_dw3x3_matches_torch(oracle_mod, B, C, H, W, seed):
    orc = oracle_mod.default()
    x, K = arrays(seed, (B, C, H, W), (C, 1, 3, 3))
    ref = F.conv2d(torch.from_numpy(x), torch.from_numpy(K), padding=1, groups=C).numpy()
    assert close(orc.dw3x3(x, K), ref)


@SETTINGS
@given(st.sampled_from([(2, 1), (2, 2), (4, 2), (6, 2), (6, 3), (8, 4), (9, 3)]),
       st.integers(1, 2), st.integers(1, 2), st.integers(0, 2 ** 31 - 1))
def test_merge_equals_sum_of_branches(oracle_mod, wk, C, n, seed):
    orc = oracle_mod.default()
    w, k = wk
    x, Tw, Tk = arrays(seed, (1, C, n * w, w), (C, (2 * w - 1) ** 2), (C, (2 * k - 1) ** 2))
    assert close(Oracle.forward_cached(x, orc.reparam_merge(Tw, Tk, w, k), w),
                 orc.forward(x, Tw, w) + orc.forward(x, Tk, k))
