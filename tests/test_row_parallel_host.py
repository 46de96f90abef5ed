"""Host side of the row-parallel layer, on the CPU: the slicing of the
input channels and of the parameters, and the identity the design rests on
(paper notes, "independent rotation": T is block diagonal over the groups),
Y = sum over ranks of (X_r T_r^-1) w_hat_r^T, checked with the fp64 oracle
on two gloo ranks that add their shares with an all-reduce."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import paro_oracle as O  # noqa: E402
from rotated_w4_linear_b200.row_parallel import shard_bounds, shard_params  # noqa: E402


@pytest.mark.parametrize("in_f,world", [(4096, 2), (4096, 8), (14336, 8), (384, 2), (256, 4)])
def test_shard_bounds_cover_on_unit_boundaries(in_f, world):
    b = shard_bounds(in_f, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == in_f
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2
    sizes = [hi - lo for lo, hi in b]
    assert all(x % 128 == 0 for x in sizes)
    assert max(sizes) - min(sizes) <= 128


def _layer(in_f=512, out_f=48, T=5, group=128, seed=21):
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=group // 2, group=group)
    q, s, z = synth.w4_codes(out_f, in_f, seed, group=group)
    x = synth.activations(T, in_f, seed)
    return x, pairs, theta, alpha, q, s, z


@pytest.mark.parametrize("group", [128, 64])
def test_shares_add_up_to_the_layer(group):
    x, pairs, theta, alpha, q, s, z = _layer(group=group)
    full = O.linear(x, pairs, theta, alpha, q, s, z, group=group)
    for world in (2, 3, 4):
        acc = np.zeros_like(full)
        for lo, hi in shard_bounds(x.shape[1], world):
            if hi == lo:
                continue
            p, t, a, qr, sr, zr = shard_params(pairs, theta, alpha, q, s, z, lo, hi, group)
            acc += O.linear(x[:, lo:hi], p, t, a, qr, sr, zr, group=group)
        assert np.allclose(acc, full, rtol=1e-12, atol=1e-12)


def test_a_cut_inside_a_group_is_refused():
    x, pairs, theta, alpha, q, s, z = _layer()
    with pytest.raises(ValueError):
        shard_params(pairs, theta, alpha, q, s, z, 0, 100, 128)
    with pytest.raises(ValueError):
        shard_bounds(500, 2)


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, pairs, theta, alpha, q, s, z = _layer(in_f=640, out_f=32, T=3)
        lo, hi = shard_bounds(640, world)[rank]
        p, t, a, qr, sr, zr = shard_params(pairs, theta, alpha, q, s, z, lo, hi)
        share = torch.from_numpy(O.linear(x[:, lo:hi], p, t, a, qr, sr, zr))
        dist.all_reduce(share, op=dist.ReduceOp.SUM)
        np.save(os.path.join(out, f"y{rank}.npy"), share.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_all_reduce_their_shares(tmp_path):
    world = 2
    mp.spawn(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    x, pairs, theta, alpha, q, s, z = _layer(in_f=640, out_f=32, T=3)
    full = O.linear(x, pairs, theta, alpha, q, s, z)
    for r in range(world):
        assert np.allclose(np.load(tmp_path / f"y{r}.npy"), full, rtol=1e-12, atol=1e-12)
