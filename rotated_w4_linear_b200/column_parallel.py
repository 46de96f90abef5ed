"""Column-parallel rotated W4 linear layer: one process per GPU, each holding
a slice of the output channels (rows of the weight).

T acts on the input channels, which every rank sees in full, so each rank
holds the whole rotation, rotates X itself and multiplies by its own rows of
w_hat (CSDN article, section 2.1, Y = (X T^-1)(T W), read per output
column):

    Y[:, lo:hi] = (X T^-1) w_hat[lo:hi]^T (+ b[lo:hi]).

The shares need no exchange; when every rank wants the whole Y, one
all-gather puts the column slices side by side. Every step on the data runs
in the library's kernels or in the collective; this module only cuts the
parameters and orders the calls. (The row-parallel form, which cuts the
input channels instead, is in row_parallel.py.)
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np

from . import binding as B

ROW_UNIT = 16      # the kernels' output unit (a row block)
TILE_UNIT = 128    # one prefill weight tile: slices start on it when the width allows


def out_bounds(out_features: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous output-channel slices [lo, hi), one per rank, cut on
    128-row boundaries when out_features allows it (else on 16-row ones),
    sizes differing by at most one unit (a rank may get none)."""
    if out_features % ROW_UNIT:
        raise ValueError(f"out_features={out_features} is not a multiple of {ROW_UNIT}")
    if world < 1:
        raise ValueError("world must be >= 1")
    unit = TILE_UNIT if out_features % TILE_UNIT == 0 else ROW_UNIT
    n = out_features // unit
    cuts = [unit * ((n * r) // world) for r in range(world + 1)]
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def out_params(q, s, z, lo: int, hi: int, bias=None):
    """Rank slice [lo, hi) of the weights' rows: q [out][in], s and z
    [out][in/group], bias [out] or None."""
    if lo % ROW_UNIT or hi % ROW_UNIT:
        raise ValueError(f"slice bounds must be multiples of {ROW_UNIT}")
    return (np.ascontiguousarray(q[lo:hi]), np.ascontiguousarray(s[lo:hi]), np.ascontiguousarray(z[lo:hi]),
            None if bias is None else np.ascontiguousarray(np.asarray(bias)[lo:hi]))


def gather_columns(Y, bounds, process_group=None):
    """The whole Y from every rank's columns: each rank passes its share
    Y [tokens][hi - lo] (a torch tensor) and the bounds of all ranks; the
    shares are padded to the widest slice (all_gather takes equal sizes),
    gathered, trimmed and put side by side in rank order."""
    import torch
    import torch.distributed as dist
    T, width = Y.shape[0], Y.shape[1]
    wmax = max(hi - lo for lo, hi in bounds)
    pad = torch.zeros((T, wmax), dtype=Y.dtype, device=Y.device)
    pad[:, :width] = Y
    parts = [torch.empty_like(pad) for _ in bounds]
    dist.all_gather(parts, pad, group=process_group)
    return torch.cat([p[:, :hi - lo] for p, (lo, hi) in zip(parts, bounds)], dim=1)


class ColumnParallelLinear:
    """This rank's part of a column-parallel layer. The parameters are given
    whole (host arrays: the rotation's pairs, theta, alpha and the logical q,
    s, z of paro_pack_weights_ex); the rank keeps the rotation and packs only
    its rows. forward() takes the whole X (fp16 CUDA tensor [tokens][in]) and
    returns the rank's columns of Y (fp16 [tokens][hi - lo]), or with
    gather=True the whole Y [tokens][out] on every rank."""

    def __init__(self, pairs, theta, alpha, q, s, z, rank: int, world: int, group: int = 128,
                 bias=None, device=None):
        import torch
        self.torch = torch
        self.out_features = int(q.shape[0])
        self.group = group
        self.bounds = out_bounds(self.out_features, world)
        self.lo, self.hi = self.bounds[rank]
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.rot = B.paro_rot_create(pairs, theta, alpha, group=group)
        self.bias = None
        if self.hi > self.lo:
            qr, sr, zr, br = out_params(q, s, z, self.lo, self.hi, bias)
            self.qw, self.sp, self.zp = B.paro_pack_weights(torch.from_numpy(qr), torch.from_numpy(sr),
                                                            torch.from_numpy(zr), device=self.device, group=group)
            if br is not None:
                self.bias = torch.as_tensor(np.asarray(br, np.float16)).to(self.device)

    def forward(self, X, process_group=None, gather: bool = False):
        torch = self.torch
        T = X.shape[0]
        width = self.hi - self.lo
        if width:
            Y = B.paro_linear_ex(self.rot, X, self.qw, self.sp, self.zp, width, group=self.group, bias=self.bias)
        else:
            Y = torch.empty((T, 0), dtype=torch.float16, device=self.device)
        if not gather:
            return Y
        import torch.distributed as dist
        if not (dist.is_available() and dist.is_initialized()):
            return Y
        return gather_columns(Y, self.bounds, process_group)

    def close(self):
        if self.rot is not None:
            self.rot.close()
            self.rot = None
