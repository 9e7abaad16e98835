"""Tolerances shared by the GPU parity tests (test infrastructure).

bf16 path (fp32 accumulation, bf16 output):
  * per element  |gpu - ref| <= 2e-2 * rowbound, rowbound the Cauchy-Schwarz
    bound of that output's dot product (||M_c[u,:]||_2 * ||X_c[:,n]||_2 for
    the forward); bf16 output rounding alone is at most 2^-9 of it;
  * whole tensor sum|gpu - ref| / sum|ref| <= 5e-3 (mean relative error as an
    L1 ratio, which stays finite where single outputs are near zero).
fp32 path: the gate is componentwise for every element,
|gpu - ref| <= 1e-5 * sum_v |M_uv x_v| (the magnitude of the output's terms,
which is never below |ref|); fp32 accumulation of d terms is bounded by
d * 2^-24 of that sum (2.9e-6 at d=49).  Beside it the check reports the plain
relative error |gpu - ref| / |ref| over the outputs with |ref| at least 1e-2
of their terms' magnitude, where it is meaningful.
"""
import numpy as np

import oracle

BF16_ROW_TOL = 2e-2
BF16_MEAN_TOL = 5e-3
F32_REL_TOL = 1e-5


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def window_norms(x, w):
    """||X_c[:, n]||_2 per window, broadcast back to [B, C, H, W]."""
    B, C, H, W = x.shape
    nh, nw = H // w, W // w
    n = np.sqrt((x.reshape(B, C, nh, w, nw, w) ** 2).sum(axis=(3, 5)))
    return np.repeat(np.repeat(n, w, axis=2), w, axis=3)


def row_norms(T, w):
    """||M_c[u, :]||_2 laid out as [C, w, w] (u = p*w + q)."""
    M = oracle.expand(T, w)
    return np.sqrt((M ** 2).sum(axis=2)).reshape(T.shape[0], w, w)


def forward_rowbound(x, T, w):
    B, C, H, W = x.shape
    rn = np.tile(row_norms(T, w), (1, H // w, W // w))
    return window_norms(x, w) * rn[None]


def check_bf16(gpu, ref, bound, what):
    err = np.abs(gpu - ref)
    worst = float(np.max(err / np.maximum(bound, 1e-30)))
    assert np.all(err <= BF16_ROW_TOL * bound + 1e-30), f"{what}: max err/rowbound {worst:.3e}"
    denom = float(np.abs(ref).sum())
    mean_rel = float(err.sum()) / denom if denom > 0 else float(err.sum())
    assert mean_rel <= BF16_MEAN_TOL, f"{what}: mean relative error {mean_rel:.3e}"
    return worst, mean_rel


def check_f32(gpu, ref, absdot, what):
    """Gate: componentwise error <= F32_REL_TOL of the terms' magnitude.
    Returns (worst componentwise error, worst plain relative error over the
    outputs with |ref| >= 1e-2 * absdot, or 0.0 if there are none)."""
    err = np.abs(gpu - ref)
    comp = err / np.maximum(np.maximum(np.abs(ref), absdot), 1e-300)
    worst = float(comp.max())
    big = np.abs(ref) >= 1e-2 * absdot
    plain = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    print("%s: componentwise %.3e, plain relative (|ref| >= 1e-2 of terms) %.3e"
          % (what, worst, plain))
    assert worst <= F32_REL_TOL, f"{what}: max componentwise error {worst:.3e}"
    return worst, plain


def dt_bound(x, dy, w):
    """Cauchy-Schwarz bound of every table-gradient bin."""
    sx = oracle.backward_dt(x * x, np.ones_like(dy), w)
    sg = oracle.backward_dt(np.ones_like(x), dy * dy, w)
    return np.sqrt(sx * sg)
