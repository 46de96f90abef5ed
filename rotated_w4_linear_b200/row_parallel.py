"""Row-parallel rotated W4 linear layer: one process per GPU, each holding a
slice of the input channels.

T is block diagonal over the quantisation groups (ParoQuant paper notes,
"independent rotation": pairs never leave their group), so with the input
channels cut on 128-channel boundaries each rank rotates only its own
channels, and

    Y = sum_r (X_r T_r^-1) w_hat_r^T (+ b),

X_r, T_r, w_hat_r being rank r's columns of X, diagonal blocks of T and
columns of the weights. Each rank computes its share as unrounded fp32 sums
(paro_linear_partial), one all-reduce (sum) over the process group adds the
shares, and paro_finalize adds the bias and rounds to fp16 once, as the
single-GPU layer does. Every step on the data runs in the library's kernels
or in the collective; this module only cuts the parameters and orders the
calls.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import numpy as np

from . import binding as B

UNIT = 128      # the kernels' channel unit: slices start and end on it


def shard_bounds(in_features: int, world: int, unit: int = UNIT) -> List[Tuple[int, int]]:
    """Contiguous input-channel slices [lo, hi), one per rank, on `unit`
    boundaries, sizes differing by at most one unit (a rank may get none
    when there are fewer units than ranks)."""
    if in_features % unit:
        raise ValueError(f"in_features={in_features} is not a multiple of {unit}")
    if world < 1:
        raise ValueError("world must be >= 1")
    n = in_features // unit
    cuts = [unit * ((n * r) // world) for r in range(world + 1)]
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def shard_params(pairs, theta, alpha, q, s, z, lo: int, hi: int, group: int = 128):
    """Rank slice [lo, hi) of the layer's parameters (group-aligned):
    pairs [K][G][P][2] and theta [K][G][P] of its groups (group-local
    indices, unchanged), alpha [in], and the columns of q [out][in] and of
    s, z [out][in/group]."""
    if lo % group or hi % group:
        raise ValueError("slice bounds must lie on group boundaries")
    g0, g1 = lo // group, hi // group
    return (np.ascontiguousarray(pairs[:, g0:g1]), np.ascontiguousarray(theta[:, g0:g1]),
            np.ascontiguousarray(alpha[lo:hi]), np.ascontiguousarray(q[:, lo:hi]),
            np.ascontiguousarray(s[:, g0:g1]), np.ascontiguousarray(z[:, g0:g1]))


class RowParallelLinear:
    """This rank's part of a row-parallel layer. The parameters are given
    whole (host arrays, the logical q, s, z of paro_pack_weights_ex); the
    rank keeps and packs only its slice. forward() takes the rank's columns of
    X (fp16 CUDA tensor [tokens][hi - lo]) and returns the whole Y (fp16
    [tokens][out]) on every rank."""

    def __init__(self, pairs, theta, alpha, q, s, z, rank: int, world: int, group: int = 128,
                 bias=None, device=None):
        import torch
        self.torch = torch
        in_features = int(alpha.shape[0])
        self.out_features = int(q.shape[0])
        self.group = group
        self.lo, self.hi = shard_bounds(in_features, world)[rank]
        self.device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.rot = None
        self.bias = None if bias is None else torch.as_tensor(np.asarray(bias, np.float16)).to(self.device)
        if self.hi > self.lo:
            p, t, a, qr, sr, zr = shard_params(pairs, theta, alpha, q, s, z, self.lo, self.hi, group)
            self.rot = B.paro_rot_create(p, t, a, group=group)
            self.qw, self.sp, self.zp = B.paro_pack_weights(torch.from_numpy(qr), torch.from_numpy(sr),
                                                            torch.from_numpy(zr), device=self.device, group=group)

    def forward(self, X_local, process_group=None):
        torch = self.torch
        import torch.distributed as dist
        T = X_local.shape[0]
        if self.rot is not None:
            Yf = B.paro_linear_partial(self.rot, X_local, self.qw, self.sp, self.zp, self.out_features,
                                       group=self.group)
        else:                                   # no channels on this rank: a zero share
            Yf = torch.zeros((T, self.out_features), dtype=torch.float32, device=self.device)
        if dist.is_available() and dist.is_initialized():
            dist.all_reduce(Yf, op=dist.ReduceOp.SUM, group=process_group)
        return B.paro_finalize(Yf, self.bias)

    def close(self):
        if self.rot is not None:
            self.rot.close()
            self.rot = None
