"""The column-parallel path on one GPU: every rank's columns of Y from
paro_linear_ex on its rows of the weights (whole X, whole rotation, its
slice of the bias), side by side, against the fp64 oracle of the whole
layer; and the host class end to end on a one-rank NCCL process group.
(Only one GPU is available per run; the multi-rank gather is tested on gloo
ranks on the CPU.)"""
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
    (5, 1024, 272, 2, 128),       # decode kernel, 16-row cuts
    (16, 4096, 1024, 4, 128),
    (300, 1536, 160, 3, 128),     # tensor-core GEMM, ragged 128-row tiles
    (12, 1024, 96, 2, 64),
    (40, 768, 256, 3, 64),
])
def test_columns_on_one_gpu(B, T, in_f, out_f, world, group):
    from rotated_w4_linear_b200.column_parallel import out_bounds, out_params
    seed = synth.layer_seed(12, T + in_f + world)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=group // 2, group=group)
    q, s, z = synth.w4_codes(out_f, in_f, seed, group=group)
    x = synth.activations(T, in_f, seed)
    b = (np.random.default_rng(seed).standard_normal(out_f) * 2).astype(np.float16)
    rot = B.paro_rot_create(pairs, theta, alpha, group=group)
    parts = []
    for lo, hi in out_bounds(out_f, world):
        if hi == lo:
            continue
        qr, sr, zr, br = out_params(q, s, z, lo, hi, b)
        qw, sp, zp = B.paro_pack_weights(dev(qr), dev(sr), dev(zr), group=group)
        parts.append(B.paro_linear_ex(rot, dev(x), qw, sp, zp, hi - lo, group=group, bias=dev(br)))
    y = torch.cat(parts, dim=1).cpu().numpy()
    check_linear(y, x, pairs, theta, alpha, q, s, z, bias=b, group=group)
    assert B.paro_fault_status() == 0


def test_host_class_on_one_nccl_rank(B):
    import torch.distributed as dist
    from rotated_w4_linear_b200.column_parallel import ColumnParallelLinear
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        T, in_f, out_f = 16, 2048, 512
        seed = synth.layer_seed(12, 1)
        pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
        q, s, z = synth.w4_codes(out_f, in_f, seed)
        x = synth.activations(T, in_f, seed)
        layer = ColumnParallelLinear(pairs, theta, alpha, q, s, z, rank=0, world=1)
        y = layer.forward(dev(x), gather=True).cpu().numpy()
        torch.cuda.synchronize()
        layer.close()
        check_linear(y, x, pairs, theta, alpha, q, s, z)
    finally:
        dist.destroy_process_group()
