"""Host side of the column-parallel layer, on the CPU: the slicing of the
output channels and of the weights' rows, the identity it rests on (each
output column needs only its own row of w_hat and the whole X T^-1; CSDN
article, section 2.1), checked with the fp64 oracle, and the gather of the
column shares on two and three gloo ranks."""
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
from rotated_w4_linear_b200.column_parallel import gather_columns, out_bounds, out_params  # noqa: E402


@pytest.mark.parametrize("out_f,world", [(6144, 2), (4096, 8), (28672, 8), (272, 2), (160, 3), (16, 4)])
def test_out_bounds_cover_on_unit_boundaries(out_f, world):
    b = out_bounds(out_f, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == out_f
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2
    unit = 128 if out_f % 128 == 0 else 16
    sizes = [hi - lo for lo, hi in b]
    assert all(x % unit == 0 for x in sizes)
    assert max(sizes) - min(sizes) <= unit


def test_bad_widths_and_cuts_are_refused():
    with pytest.raises(ValueError):
        out_bounds(100, 2)
    q = np.zeros((64, 128), np.uint8)
    s = np.ones((64, 1), np.float16)
    with pytest.raises(ValueError):
        out_params(q, s, q[:, :1], 0, 40)


def _layer(in_f=512, out_f=160, T=5, group=128, seed=31):
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=group // 2, group=group)
    q, s, z = synth.w4_codes(out_f, in_f, seed, group=group)
    x = synth.activations(T, in_f, seed)
    b = (np.random.default_rng(seed).standard_normal(out_f) * 2).astype(np.float16)
    return x, pairs, theta, alpha, q, s, z, b


@pytest.mark.parametrize("group", [128, 64])
def test_column_shares_are_the_layer_columns(group):
    x, pairs, theta, alpha, q, s, z, b = _layer(group=group)
    full = O.linear(x, pairs, theta, alpha, q, s, z, group=group, bias=b)
    for world in (2, 3, 4):
        parts = []
        for lo, hi in out_bounds(q.shape[0], world):
            qr, sr, zr, br = out_params(q, s, z, lo, hi, b)
            parts.append(O.linear(x, pairs, theta, alpha, qr, sr, zr, group=group, bias=br))
        assert np.allclose(np.concatenate(parts, axis=1), full, rtol=1e-12, atol=1e-12)


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, pairs, theta, alpha, q, s, z, b = _layer(out_f=160, T=3)
        bounds = out_bounds(160, world)
        lo, hi = bounds[rank]
        qr, sr, zr, br = out_params(q, s, z, lo, hi, b)
        share = torch.from_numpy(O.linear(x, pairs, theta, alpha, qr, sr, zr, bias=br))
        np.save(os.path.join(out, f"y{rank}.npy"), gather_columns(share, bounds).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_their_columns(tmp_path, world):
    mp.spawn(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    x, pairs, theta, alpha, q, s, z, b = _layer(out_f=160, T=3)
    full = O.linear(x, pairs, theta, alpha, q, s, z, bias=b)
    for r in range(world):
        assert np.allclose(np.load(tmp_path / f"y{r}.npy"), full, rtol=1e-12, atol=1e-12)
