"""Seeded input generator: determinism, shapes, dtypes and the truncation rule."""
import torch

import synth


def test_draw_is_deterministic_and_shaped():
    wl = synth.WORKLOADS["tiny_fp32"]
    a, b = synth.draw(wl, seed=0), synth.draw(wl, seed=0)
    assert set(a) == {"x", "T"}
    assert torch.equal(a["x"], b["x"]) and torch.equal(a["T"], b["T"])
    assert a["x"].shape == (1, 4, 14, 14) and a["T"].shape == (4, 169)
    assert a["x"].dtype == torch.float32
    c = synth.draw(wl, seed=1)
    assert not torch.equal(a["x"], c["x"])


def test_truncated_table_and_kinds():
    wl = synth.WORKLOADS["train_bf16"].scaled(B=2, C=8)
    d = synth.draw(wl, seed=0)
    assert set(d) == {"x", "T", "dY"}
    assert d["x"].dtype == torch.bfloat16 and d["T"].dtype == torch.bfloat16
    assert float(d["T"].float().abs().max()) <= 2 * synth.TABLE_SIGMA * (1 + 2 ** -8)
    wl5 = synth.WORKLOADS["hires_cached_dw"].scaled(B=1, C=4, H=28, W=28)
    d5 = synth.draw(wl5, seed=0)
    assert set(d5) == {"x", "T", "K"} and d5["K"].shape == (4, 1, 3, 3)


def test_workload_table():
    w = synth.WORKLOADS
    assert (w["fwd_bf16"].d, w["fwd_bf16"].windows_per_channel) == (196, 1024)
    assert w["train_bf16"].windows_per_channel == 512
    assert w["hires_cached_dw"].windows_per_channel == 2048
    assert w["sweep_w28"].t == 55 * 55
