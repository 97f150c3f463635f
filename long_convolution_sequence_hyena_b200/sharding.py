"""Channel partition of the operator over ranks (one process per GPU).

The operator is depthwise: every (b, d) row (every (b, c) plane in 2D) is an
independent problem, and channel d only ever reads its own filter rows
h^n[d] and feedthroughs Dskip^n_d ("Hyena, Long Convolution, and Linear
Attention", "FFTConv": one filter per channel). Splitting the channels into
contiguous ranges therefore needs no collective on the data path: a rank
takes its slice of v, of every gate and of y, builds a plan for its channel
count, and computes the spectra of its own filter rows only.
"""
from __future__ import annotations


def channel_range(channels: int, world: int, rank: int) -> tuple[int, int]:
    """[d0, d1) of `rank` among `world` ranks: contiguous, sizes differ by at most one,
    the first `channels % world` ranks take one extra channel."""
    if world < 1 or not 0 <= rank < world or channels < 0:
        raise ValueError("bad partition: channels=%d world=%d rank=%d" % (channels, world, rank))
    base, extra = divmod(channels, world)
    d0 = rank * base + min(rank, extra)
    return d0, d0 + base + (1 if rank < extra else 0)


def shard_inputs(inputs: dict, d0: int, d1: int) -> dict:
    """A rank's slice of the operator's tensors: v [B, D, ...], gates [N, B, D, ...] (or a list of
    [B, D, ...]), filters h [N, D, ...], dskip [N, D]. Slices are views (no copy)."""
    out = dict(inputs)
    n = d1 - d0
    out["v"] = inputs["v"].narrow(1, d0, n)
    g = inputs["gates"]
    out["gates"] = [x.narrow(1, d0, n) for x in g] if isinstance(g, (list, tuple)) else g.narrow(2, d0, n)
    if "h" in inputs:
        out["h"] = inputs["h"].narrow(1, d0, n)
    if inputs.get("dskip") is not None:
        out["dskip"] = inputs["dskip"].narrow(1, d0, n)
    return out
