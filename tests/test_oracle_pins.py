"""Pins for the WBMM oracle: checks against things other than the oracle itself.

Each pin ties an oracle function to a library routine (torch conv2d), a closed
form, an exact special case or an invariant fixed by the mathematics of the
operator.  The planted-mistake tests at the bottom compile copies of the
oracle with one deliberate bug each and show that some pin catches it.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import Oracle


def rnd(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def center(w):
    return (w - 1) * (2 * w - 1) + (w - 1)


def table_from_kernel(K, w):
    """Table whose WBMM equals a k x k cross-correlation inside each window.

    Reading: a torch conv2d weight K[a, e] (a, e in 0..k-1, padding k//2)
    reaches input (p + a - k//2, q + e - k//2) from output (p, q), i.e. the
    offset p - r = k//2 - a; so T[(w-1+k//2-a)(2w-1) + (w-1+k//2-e)] = K[a, e].
    """
    C, k, _ = K.shape
    T = np.zeros((C, (2 * w - 1) ** 2))
    h = k // 2
    for a in range(k):
        for e in range(k):
            T[:, (w - 1 + h - a) * (2 * w - 1) + (w - 1 + h - e)] = K[:, a, e]
    return T


def windows_as_images(x, w):
    """[B,C,H,W] -> [B*nh*nw, C, w, w]: every window as its own image."""
    B, C, H, W = x.shape
    nh, nw = H // w, W // w
    return x.reshape(B, C, nh, w, nw, w).transpose(0, 2, 4, 1, 3, 5).reshape(B * nh * nw, C, w, w)


def images_as_map(xw, B, C, H, W, w):
    nh, nw = H // w, W // w
    return xw.reshape(B, nh, nw, C, w, w).transpose(0, 3, 1, 4, 2, 5).reshape(B, C, H, W)


# --------------------------------------------------------------------------
# Forward pins
# --------------------------------------------------------------------------

def pin_identity(orc):
    for w in (1, 2, 3, 7, 14):
        x = rnd((2, 3, 2 * w, 3 * w), 10 + w)
        T = np.zeros((3, (2 * w - 1) ** 2))
        T[:, center(w)] = 1.0
        assert np.array_equal(orc.forward(x, T, w), x)


def pin_shift(orc):
    # one-hot table at offset (dp, dq): y[p,q] = x[p-dp, q-dq] inside the window, else 0
    w = 5
    x = rnd((2, 2, 10, 15), 3)
    for dp, dq in [(1, 0), (0, 2), (-3, 1), (4, -4), (-1, -2)]:
        T = np.zeros((2, 81))
        T[:, (dp + w - 1) * (2 * w - 1) + (dq + w - 1)] = 1.0
        y = orc.forward(x, T, w)
        xw = windows_as_images(x, w)
        ew = np.zeros_like(xw)
        for p in range(w):
            for q in range(w):
                r, s = p - dp, q - dq
                if 0 <= r < w and 0 <= s < w:
                    ew[:, :, p, q] = xw[:, :, r, s]
        assert np.array_equal(y, images_as_map(ew, 2, 2, 10, 15, w)), (dp, dq)


def pin_constant_table(orc):
    w = 4
    x = rnd((3, 2, 8, 12), 5)
    T = np.ones((2, 49))
    y = orc.forward(x, T, w)
    xw = windows_as_images(x, w)
    sums = xw.sum(axis=(2, 3), keepdims=True) * np.ones_like(xw)
    np.testing.assert_allclose(y, images_as_map(sums, 3, 2, 8, 12, w), rtol=1e-13, atol=1e-13)


def pin_conv_equivalence(orc):
    # k x k depthwise cross-correlation (torch, fp64) applied to each window as
    # its own zero-padded image equals WBMM with the matching table.
    cases = [(3, 3), (3, 5), (7, 1), (7, 3), (7, 5), (7, 7), (14, 3), (14, 5), (14, 7)]
    for w, k in cases:
        B, C, H, W = 2, 3, 2 * w, 2 * w
        x = rnd((B, C, H, W), 100 + w * k)
        K = rnd((C, k, k), 200 + w * k)
        T = table_from_kernel(K, w)
        y = orc.forward(x, T, w)
        xw = torch.from_numpy(windows_as_images(x, w))
        ref = F.conv2d(xw, torch.from_numpy(K).unsqueeze(1), padding=k // 2, groups=C).numpy()
        np.testing.assert_allclose(y, images_as_map(ref, B, C, H, W, w),
                                   rtol=1e-12, atol=1e-12, err_msg=f"w={w} k={k}")


def pin_window_locality(orc):
    w = 4
    x = rnd((2, 2, 8, 12), 7)
    T = rnd((2, 49), 8)
    y0 = orc.forward(x, T, w)
    x1 = x.copy()
    x1[1, 0, 4:8, 4:8] += rnd((4, 4), 9)          # window (b=1, c=0, i=1, j=1)
    diff = orc.forward(x1, T, w) - y0
    mask = np.zeros_like(diff, dtype=bool)
    mask[1, 0, 4:8, 4:8] = True
    assert np.all(diff[~mask] == 0.0)
    assert np.any(diff[mask] != 0.0)


def pin_batch_permutation(orc):
    w = 3
    x = rnd((4, 2, 6, 9), 11)
    T = rnd((2, 25), 12)
    perm = [2, 0, 3, 1]
    assert np.array_equal(orc.forward(x[perm], T, w), orc.forward(x, T, w)[perm])


def _worked_example():
    path = os.path.join(os.path.dirname(__file__), "golden", "worked_example_w2.txt")
    g = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            g[k] = np.array([float(t) for t in v])
    return g


def pin_worked_example(orc):
    # hand-computed values (tests/golden/worked_example_w2.txt) pin the index
    # convention, the window layout, both gradients, the cached matrix and the
    # 3x3 mixing to numbers
    g, w = _worked_example(), 2
    x, T, dy = g["x"].reshape(1, 1, 2, 4), g["T"].reshape(1, 9), g["dY"].reshape(1, 1, 2, 4)
    y = orc.forward(x, T, w)
    assert np.array_equal(y.reshape(-1), g["y"])
    assert np.array_equal(orc.backward_dx(dy, T, w).reshape(-1), g["dX"])
    assert np.array_equal(orc.backward_dt(x, dy, w).reshape(-1), g["dT"])
    assert np.array_equal(orc.expand(T, w).reshape(-1), g["M"])
    assert np.array_equal(orc.dw3x3(g["y"].reshape(1, 1, 2, 4), g["K"].reshape(1, 1, 3, 3))
                          .reshape(-1), g["z"])
    assert np.array_equal(orc.reparam_merge(T, g["Tk"].reshape(1, 1), w, 1).reshape(-1),
                          g["Mmerged"])


FORWARD_PINS = [pin_identity, pin_shift, pin_constant_table, pin_conv_equivalence,
                pin_window_locality, pin_batch_permutation, pin_worked_example]


# --------------------------------------------------------------------------
# Gradient pins
# --------------------------------------------------------------------------

def pin_dx_adjoint(orc):
    for w in (2, 5, 7):
        x = rnd((2, 3, 2 * w, 3 * w), 20 + w)
        dy = rnd(x.shape, 30 + w)
        T = rnd((3, (2 * w - 1) ** 2), 40 + w)
        lhs = np.sum(dy * orc.forward(x, T, w))
        rhs = np.sum(orc.backward_dx(dy, T, w) * x)
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), (w, lhs, rhs)


def pin_dx_finite_difference(orc):
    # L(x) = <dY, WBMM(x)> is linear in x, so the central difference with
    # eps = 1 is exact up to rounding: dL/dx_i = dX_i.
    w = 7
    x = rnd((1, 4, 14, 14), 50)          # the tiny fp32 workload's shape
    dy = rnd(x.shape, 51)
    T = rnd((4, 169), 52, 0.02)
    dx = orc.backward_dx(dy, T, w)
    g = np.random.default_rng(53)
    for _ in range(40):
        idx = tuple(int(g.integers(0, s)) for s in x.shape)
        xp, xm = x.copy(), x.copy()
        xp[idx] += 1.0
        xm[idx] -= 1.0
        fd = (np.sum(dy * orc.forward(xp, T, w)) - np.sum(dy * orc.forward(xm, T, w))) / 2.0
        assert abs(fd - dx[idx]) <= 1e-10 * max(1.0, abs(fd)), (idx, fd, dx[idx])


def pin_dt_finite_difference(orc):
    w = 7
    x = rnd((1, 4, 14, 14), 60)
    dy = rnd(x.shape, 61)
    T = rnd((4, 169), 62, 0.02)
    dT = orc.backward_dt(x, dy, w)
    g = np.random.default_rng(63)
    for _ in range(40):
        c, k = int(g.integers(0, 4)), int(g.integers(0, 169))
        Tp, Tm = T.copy(), T.copy()
        Tp[c, k] += 1.0
        Tm[c, k] -= 1.0
        fd = (np.sum(dy * orc.forward(x, Tp, w)) - np.sum(dy * orc.forward(x, Tm, w))) / 2.0
        assert abs(fd - dT[c, k]) <= 1e-10 * max(1.0, abs(fd)), (c, k, fd, dT[c, k])


def pin_dt_adjoint(orc):
    w = 4
    x = rnd((3, 2, 8, 12), 70)
    dy = rnd(x.shape, 71)
    dTdir = rnd((2, 49), 72)
    lhs = np.sum(orc.backward_dt(x, dy, w) * dTdir)
    rhs = np.sum(dy * orc.forward(x, dTdir, w))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def pin_dt_count_closed_form(orc):
    # x = dY = 1: each bin counts its pairs, N_c (w-|dp|)(w-|dq|).
    for w in (2, 3, 14):
        B, C, H, W = 2, 2, 2 * w, w
        Nc = B * (H // w) * (W // w)
        dT = orc.backward_dt(np.ones((B, C, H, W)), np.ones((B, C, H, W)), w)
        exp = np.array([[Nc * (w - abs(dp)) * (w - abs(dq))
                         for dp in range(-w + 1, w) for dq in range(-w + 1, w)]] * C, float)
        assert np.array_equal(dT, exp)
        assert dT[0].sum() == Nc * w ** 4
    # sum over offsets of (w-|dp|)(w-|dq|) is d^2: 38416 at w = 14
    assert sum((14 - abs(a)) * (14 - abs(b)) for a in range(-13, 14) for b in range(-13, 14)) == 38416


def pin_dt_sum_invariant(orc):
    # sum_t dT_c[t] = sum over windows of (sum_u dY)(sum_v X)
    w = 3
    x = rnd((2, 3, 6, 9), 80)
    dy = rnd(x.shape, 81)
    dT = orc.backward_dt(x, dy, w)
    xs = windows_as_images(x, w).sum(axis=(2, 3))
    gs = windows_as_images(dy, w).sum(axis=(2, 3))
    np.testing.assert_allclose(dT.sum(axis=1), (xs * gs).sum(axis=0), rtol=1e-12, atol=1e-12)


GRADIENT_PINS = [pin_dx_adjoint, pin_dx_finite_difference, pin_dt_finite_difference,
                 pin_dt_adjoint, pin_dt_count_closed_form, pin_dt_sum_invariant,
                 pin_worked_example]


# --------------------------------------------------------------------------
# Expansion, cached path, 3x3 mixing
# --------------------------------------------------------------------------

def pin_expand(orc):
    w = 3
    Tid = np.zeros((2, 25))
    Tid[:, center(w)] = 1.0
    assert np.array_equal(orc.expand(Tid, w), np.broadcast_to(np.eye(9), (2, 9, 9)))
    # an expanded matrix applied by a library matmul reproduces the forward
    for w in (2, 5, 7):
        x = rnd((2, 3, 2 * w, w), 90 + w)
        T = rnd((3, (2 * w - 1) ** 2), 91 + w)
        np.testing.assert_allclose(Oracle.forward_cached(x, orc.expand(T, w), w),
                                   orc.forward(x, T, w), rtol=1e-12, atol=1e-12)


def pin_dw3x3(orc):
    x = rnd((2, 5, 9, 13), 95)
    K = rnd((5, 1, 3, 3), 96)
    ref = F.conv2d(torch.from_numpy(x), torch.from_numpy(K), padding=1, groups=5).numpy()
    np.testing.assert_allclose(orc.dw3x3(x, K), ref, rtol=1e-12, atol=1e-12)


def pin_reparam_merge(orc):
    # no small branch: the expansion of the big table (pinned above)
    Tw = rnd((2, 49), 97)
    assert np.array_equal(orc.reparam_merge(Tw, np.zeros((2, 9)), 4, 2), orc.expand(Tw, 4))
    # equal windows: the tables simply add
    Tk = rnd((2, 49), 98)
    np.testing.assert_allclose(orc.reparam_merge(Tw, Tk, 4, 4), orc.expand(Tw + Tk, 4),
                               rtol=1e-15, atol=1e-15)
    # the folded matrix computes the sum of the two branches: a w-window WBMM
    # and a k-window WBMM on the same map
    for w, k in ((4, 2), (6, 3), (6, 2), (14, 7)):
        x = rnd((2, 3, 2 * w, w), 100 + w + k)
        Tw = rnd((3, (2 * w - 1) ** 2), 101 + w)
        Tk = rnd((3, (2 * k - 1) ** 2), 102 + k)
        np.testing.assert_allclose(Oracle.forward_cached(x, orc.reparam_merge(Tw, Tk, w, k), w),
                                   orc.forward(x, Tw, w) + orc.forward(x, Tk, k),
                                   rtol=1e-12, atol=1e-12)


OTHER_PINS = [pin_expand, pin_dw3x3, pin_reparam_merge, pin_worked_example]
ALL_PINS = list(dict.fromkeys(FORWARD_PINS + GRADIENT_PINS + OTHER_PINS))


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_mod):
    pin(oracle_mod.default())


def test_dx_is_forward_with_rotated_table(oracle_mod):
    # Reading used by the CUDA path: M_c^T is the matrix of the 180-degree
    # rotated table, T'[k] = T[t-1-k]; the oracle's adjoint loop agrees.
    orc = oracle_mod.default()
    for w in (3, 7):
        dy = rnd((2, 2, 2 * w, 2 * w), 300 + w)
        T = rnd((2, (2 * w - 1) ** 2), 301 + w)
        np.testing.assert_allclose(orc.backward_dx(dy, T, w), orc.forward(dy, T[:, ::-1], w),
                                   rtol=1e-12, atol=1e-12)


def test_cached_forward_accepts_any_matrix(oracle_mod):
    # forward_cached is the plain product: a random M against an explicit loop.
    w = 2
    x = rnd((1, 2, 2, 4), 310)
    M = rnd((2, 4, 4), 311)
    y = Oracle.forward_cached(x, M, w)
    for c in range(2):
        for j in range(2):
            win = x[0, c, :, 2 * j:2 * j + 2].reshape(4)
            np.testing.assert_allclose(y[0, c, :, 2 * j:2 * j + 2].reshape(4), M[c] @ win,
                                       rtol=1e-14, atol=1e-14)


def test_receptive_field_golden():
    path = os.path.join(os.path.dirname(__file__), "golden", "receptive_field.txt")
    vals = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    ratio = vals["window"] ** 2 / vals["kernel"] ** 2
    assert ratio == pytest.approx(7.84)
    assert round(ratio, 1) == vals["stated_ratio"]


def test_oracle_rejects_bad_shapes(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.forward(np.zeros((1, 1, 5, 6)), np.zeros((1, 9)), 2)
    with pytest.raises(ValueError):
        oracle_mod.forward(np.zeros((1, 2, 4, 4)), np.zeros((1, 9)), 2)


# --------------------------------------------------------------------------
# Planted mistakes: each compiled mutant of the oracle must fail some pin.
# --------------------------------------------------------------------------

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "wbmm_oracle.c")

# (name, function whose body is mutated, old text, new text, pin group)
MUTANTS = [
    ("fwd_transposed_offset", "oracle_forward", "rel_index(w, p - r, q - s)",
     "rel_index(w, q - s, p - r)", FORWARD_PINS),
    ("fwd_wrong_sign", "oracle_forward", "rel_index(w, p - r, q - s)",
     "rel_index(w, r - p, s - q)", FORWARD_PINS),
    ("fwd_dropped_last_column", "oracle_forward", "for (int s = 0; s < w; ++s)",
     "for (int s = 0; s < w - 1; ++s)", FORWARD_PINS),
    ("fwd_window_origin", "oracle_forward", "[(long)(i * w + r) * W + j * w + s]",
     "[(long)(i * w + r) * W + j * w + (s + 1) % w]", FORWARD_PINS),
    ("dx_not_transposed", "oracle_backward_dx", "rel_index(w, p - r, q - s)",
     "rel_index(w, r - p, s - q)", GRADIENT_PINS),
    ("dx_swapped_axes", "oracle_backward_dx", "rel_index(w, p - r, q - s)",
     "rel_index(w, q - s, p - r)", GRADIENT_PINS),
    ("dt_wrong_bin", "oracle_backward_dt", "g[rel_index(w, p - r, q - s)]",
     "g[rel_index(w, r - p, q - s)]", GRADIENT_PINS),
    ("dt_dropped_pairs", "oracle_backward_dt", "for (int r = 0; r < w; ++r)",
     "for (int r = 1; r < w; ++r)", GRADIENT_PINS),
    ("dw_flipped_kernel", "oracle_dw3x3", "Kc[a * 3 + e]", "Kc[e * 3 + a]", OTHER_PINS),
    ("dw_shifted_row", "oracle_dw3x3", "const int hh = h + a - 1", "const int hh = h + a - 2",
     OTHER_PINS),
    ("rp_row_blocks_only", "oracle_reparam_merge", "p / k == r / k && q / k == s / k",
     "p / k == r / k", OTHER_PINS),
    ("rp_transposed_small", "oracle_reparam_merge",
     "rel_index(k, p % k - r % k, q % k - s % k)", "rel_index(k, q % k - s % k, p % k - r % k)",
     OTHER_PINS),
    ("rp_flipped_small", "oracle_reparam_merge",
     "rel_index(k, p % k - r % k, q % k - s % k)", "rel_index(k, r % k - p % k, s % k - q % k)",
     OTHER_PINS),
]


def _mutate(src, func, old, new):
    start = src.index("void " + func + "(")
    end = src.index("\n}\n", start)
    body = src[start:end]
    assert old in body, (func, old)
    return src[:start] + body.replace(old, new) + src[end:]


def _compile_mutant(src, tmpdir, name):
    c_path = os.path.join(tmpdir, name + ".c")
    so_path = os.path.join(tmpdir, name + ".so")
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so_path,
                    c_path], check=True, capture_output=True)
    return Oracle(so_path)


def _fails_some(pins, orc):
    for pin in pins:
        try:
            pin(orc)
        except AssertionError:
            return pin.__name__
    return None


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m[0])
def test_planted_mistake_is_caught(mutant):
    name, func, old, new, pins = mutant
    src = open(ORACLE_SRC).read()
    with tempfile.TemporaryDirectory() as td:
        orc = _compile_mutant(_mutate(src, func, old, new), td, name)
        caught = _fails_some(pins, orc)
    assert caught is not None, f"no pin caught the planted mistake {name}"

