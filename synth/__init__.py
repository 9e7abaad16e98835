"""Seeded synthetic inputs for WBMM workloads.

This module holds only random-number draws and the workload shapes; it does
none of the operator's arithmetic.  Both the oracle-based tests and the CUDA
path's tests/benchmark take their inputs from here, so the two sides always
see identical stored values.

Draw recipe (one CPU ``torch.Generator`` seeded once, fixed draw order):
  1. x  ~ N(0, 1)                      shape [B, C, H, W]
  2. T  ~ N(0, 0.02^2)                 shape [C, (2w-1)^2]; "truncated" tables
                                        redraw every entry with |T| > 2 sigma
                                        until none is left
  3. dY ~ N(0, 1)                      shape [B, C, H, W]   (training workloads)
  4. K  ~ N(0, 1/9)                    shape [C, 1, 3, 3]   (3x3 mixing weights)
  5. Tk ~ N(0, 0.02^2)                 shape [C, (2k-1)^2]  (second-branch table of
                                        the reparameterisation workloads, k = 7)
All values are drawn in fp32 and then cast (round to nearest even) to the
workload's dtype; the cast values are the inputs of record.
"""
from dataclasses import dataclass, replace

import torch

TABLE_SIGMA = 0.02
DW_SIGMA = 1.0 / 3.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    C: int
    H: int
    W: int
    w: int
    dtype: str          # "f32" or "bf16"
    table: str          # "normal" or "truncated"
    kind: str           # "forward", "train", "cached_dw" or "reparam"

    @property
    def d(self):
        return self.w * self.w

    @property
    def t(self):
        return (2 * self.w - 1) ** 2

    @property
    def windows_per_channel(self):
        return self.B * (self.H // self.w) * (self.W // self.w)

    def scaled(self, **kw):
        return replace(self, **kw)


# The five workloads of the operator benchmark (the w-sweep counts as three).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 4, 14, 14, 7, "f32", "normal", "forward"),
    "fwd_bf16": Workload("fwd_bf16", 64, 128, 56, 56, 14, "bf16", "truncated", "forward"),
    "fwd_f32": Workload("fwd_f32", 64, 128, 56, 56, 14, "f32", "truncated", "forward"),
    "train_bf16": Workload("train_bf16", 128, 256, 28, 28, 14, "bf16", "truncated", "train"),
    "sweep_w7": Workload("sweep_w7", 32, 256, 112, 112, 7, "bf16", "normal", "forward"),
    "sweep_w14": Workload("sweep_w14", 32, 256, 112, 112, 14, "bf16", "normal", "forward"),
    "sweep_w28": Workload("sweep_w28", 32, 256, 112, 112, 28, "bf16", "normal", "forward"),
    "hires_cached_dw": Workload("hires_cached_dw", 8, 96, 224, 224, 14, "bf16", "normal",
                                "cached_dw"),
    # the fp32 path (CUDA cores) on the training and high-res cached shapes
    "train_f32": Workload("train_f32", 128, 256, 28, 28, 14, "f32", "truncated", "train"),
    "hires_cached_dw_f32": Workload("hires_cached_dw_f32", 8, 96, 224, 224, 14, "f32", "normal",
                                    "cached_dw"),
    # inference with a 14x14 and a 7x7 branch folded into one matrix
    "hires_reparam": Workload("hires_reparam", 8, 96, 224, 224, 14, "bf16", "normal", "reparam"),
}

# second branch window of the "reparam" workloads
REPARAM_SMALL_WINDOW = 7


def torch_dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _truncated_normal(gen, shape, sigma):
    v = torch.randn(shape, generator=gen, dtype=torch.float32) * sigma
    while True:
        bad = v.abs() > 2.0 * sigma
        n = int(bad.sum())
        if n == 0:
            return v
        v[bad] = torch.randn(n, generator=gen, dtype=torch.float32) * sigma


def draw(wl: Workload, seed: int = 0):
    """Return a dict of CPU tensors (x, T and, by kind, dY / K) for ``wl``."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    dt = torch_dtype(wl.dtype)
    out = {}
    out["x"] = torch.randn((wl.B, wl.C, wl.H, wl.W), generator=gen,
                           dtype=torch.float32).to(dt)
    if wl.table == "truncated":
        T = _truncated_normal(gen, (wl.C, wl.t), TABLE_SIGMA)
    else:
        T = torch.randn((wl.C, wl.t), generator=gen, dtype=torch.float32) * TABLE_SIGMA
    out["T"] = T.to(dt)
    if wl.kind == "train":
        out["dY"] = torch.randn((wl.B, wl.C, wl.H, wl.W), generator=gen,
                                dtype=torch.float32).to(dt)
    if wl.kind == "cached_dw":
        out["K"] = (torch.randn((wl.C, 1, 3, 3), generator=gen, dtype=torch.float32)
                    * DW_SIGMA).to(dt)
    if wl.kind == "reparam":
        k = REPARAM_SMALL_WINDOW
        out["Tk"] = (torch.randn((wl.C, (2 * k - 1) ** 2), generator=gen, dtype=torch.float32)
                     * TABLE_SIGMA).to(dt)
    return out


def draw_tensor(shape, seed, dtype="f32", sigma=1.0):
    """One seeded N(0, sigma^2) tensor, for ad-hoc test inputs."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * sigma).to(torch_dtype(dtype))
