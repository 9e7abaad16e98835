"""Channel sharding for multi-GPU runs.

WBMM's channels are independent (T_c, X_c, Y_c and dT_c touch no other
channel), so N processes split the channel axis into contiguous blocks and
need no collective on the data path.  Pure host logic: no device work.
"""


def channel_range(total_channels, world, rank):
    """[c0, c1): the contiguous channel block of `rank`; blocks differ by at most one."""
    if world < 1 or not 0 <= rank < world or total_channels < 0:
        raise ValueError("bad world/rank/channels")
    q, r = divmod(total_channels, world)
    c0 = rank * q + min(rank, r)
    return c0, c0 + q + (1 if rank < r else 0)


def local_channels(t, world, rank, dim=1):
    """The slice of tensor/array `t` along `dim` that `rank` owns."""
    c0, c1 = channel_range(t.shape[dim], world, rank)
    index = [slice(None)] * t.ndim
    index[dim] = slice(c0, c1)
    return t[tuple(index)]
