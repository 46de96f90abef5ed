"""The row-parallel path on one GPU: rank shares from paro_linear_partial
(unrounded fp32 sums over each input slice), added, then paro_finalize
(bias, one rounding), against the fp64 oracle of the whole layer; and the
host class end to end on a one-rank NCCL process group. (Only one GPU is
available per run; the multi-rank logic is tested on gloo ranks on the CPU.)"""
import os
import socket

import numpy as np
import pytest
import torch

import synth
from parity import check_linear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_lib):
    from rotated_w4_linear_b200 import binding
    return binding


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("T,in_f,out_f,world,group", [
    (5, 1024, 272, 2, 128),       # decode kernel
    (16, 4096, 1024, 4, 128),
    (300, 1536, 160, 3, 128),     # tensor-core GEMM
    (12, 1024, 96, 2, 64),
    (40, 768, 48, 2, 64),
])
def test_shares_on_one_gpu(B, T, in_f, out_f, world, group):
    from rotated_w4_linear_b200.row_parallel import shard_bounds, shard_params
    seed = synth.layer_seed(11, T + in_f + world)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=group // 2, group=group)
    q, s, z = synth.w4_codes(out_f, in_f, seed, group=group)
    x = synth.activations(T, in_f, seed)
    b = (np.random.default_rng(seed).standard_normal(out_f) * 2).astype(np.float16)
    total = torch.zeros((T, out_f), dtype=torch.float32, device="cuda")
    for lo, hi in shard_bounds(in_f, world):
        p, t, a, qr, sr, zr = shard_params(pairs, theta, alpha, q, s, z, lo, hi, group)
        rot = B.paro_rot_create(p, t, a, group=group)
        qw, sp, zp = B.paro_pack_weights(dev(qr), dev(sr), dev(zr), group=group)
        total += B.paro_linear_partial(rot, dev(x[:, lo:hi]), qw, sp, zp, out_f, group=group)
    y = B.paro_finalize(total, dev(b)).cpu().numpy()
    check_linear(y, x, pairs, theta, alpha, q, s, z, bias=b, group=group)
    assert B.paro_fault_status() == 0


def test_host_class_on_one_nccl_rank(B):
    import torch.distributed as dist
    from rotated_w4_linear_b200.row_parallel import RowParallelLinear
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        T, in_f, out_f = 16, 2048, 512
        seed = synth.layer_seed(11, 1)
        pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
        q, s, z = synth.w4_codes(out_f, in_f, seed)
        x = synth.activations(T, in_f, seed)
        layer = RowParallelLinear(pairs, theta, alpha, q, s, z, rank=0, world=1)
        y = layer.forward(dev(x)).cpu().numpy()
        torch.cuda.synchronize()
        layer.close()
        check_linear(y, x, pairs, theta, alpha, q, s, z)
    finally:
        dist.destroy_process_group()
