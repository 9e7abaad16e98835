"""Multi-process channel sharding on CPU (gloo, world size 2).

Each rank takes its channel block of one global seeded problem, computes the
forward and the table gradient of its block (with the oracle: these are CPU
processes), and the ranks all-gather the blocks.  The gathered result must
equal the single-process result exactly: the channel split needs no exchange
on the data path.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from windowed_matmul_conv_b200.sharding import channel_range, local_channels
        wl = synth.WORKLOADS["train_bf16"].scaled(B=2, C=5, H=28, W=28)
        d = synth.draw(wl, seed=0)
        c0, c1 = channel_range(wl.C, world, rank)
        x = local_channels(d["x"], world, rank).float()
        dy = local_channels(d["dY"], world, rank).float()
        T = d["T"][c0:c1].float()
        y = torch.from_numpy(oracle.forward(x, T, wl.w))
        dT = torch.from_numpy(oracle.backward_dt(x, dy, wl.w))
        # blocks differ by at most one channel: pad to the largest for the gather
        cmax = channel_range(wl.C, world, 0)[1]
        yp = torch.zeros((wl.B, cmax, wl.H, wl.W), dtype=torch.float64)
        yp[:, : c1 - c0] = y
        dTp = torch.zeros((cmax, wl.t), dtype=torch.float64)
        dTp[: c1 - c0] = dT
        ys = [torch.empty_like(yp) for _ in range(world)]
        dTs = [torch.empty_like(dTp) for _ in range(world)]
        dist.all_gather(ys, yp)
        dist.all_gather(dTs, dTp)
        if rank == 0:
            parts_y, parts_t = [], []
            for r in range(world):
                a, b = channel_range(wl.C, world, r)
                parts_y.append(ys[r][:, : b - a])
                parts_t.append(dTs[r][: b - a])
            torch.save({"y": torch.cat(parts_y, 1), "dT": torch.cat(parts_t, 0)},
                       os.path.join(out_dir, "gathered.pt"))
    finally:
        dist.destroy_process_group()


def test_channel_range_partitions():
    from windowed_matmul_conv_b200.sharding import channel_range
    for total in (1, 5, 128, 257):
        for world in (1, 2, 3, 8):
            blocks = [channel_range(total, world, r) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == total
            assert all(blocks[i][1] == blocks[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_channel_sharding_matches_single_process(tmp_path):
    import oracle
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = torch.load(os.path.join(tmp_path, "gathered.pt"))
    wl = synth.WORKLOADS["train_bf16"].scaled(B=2, C=5, H=28, W=28)
    d = synth.draw(wl, seed=0)
    y = oracle.forward(d["x"], d["T"], wl.w)
    dT = oracle.backward_dt(d["x"], d["dY"], wl.w)
    assert np.array_equal(got["y"].numpy(), y)
    assert np.array_equal(got["dT"].numpy(), dT)
