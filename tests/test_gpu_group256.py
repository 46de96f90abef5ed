"""Groups of 256 channels (the accuracy end of the group-size knob, CSDN
article, section 5.2): rotation pairs anywhere inside 256-channel groups (the
tensor-core rotation with 256 x 256 matrices serves every batch size) and
W4G256 weights (stored in the group-128 format with each scale and zero
repeated), through the C ABI, against the fp64 oracle run with group = 256."""
import numpy as np
import pytest
import torch

import synth
from oracle import paro_oracle as O
from parity import check_linear, check_rotation

pytestmark = pytest.mark.gpu
G256 = 256


@pytest.fixture(scope="module")
def B(cuda_lib):
    from rotated_w4_linear_b200 import binding
    return binding


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("T,in_f,K,P", [(1, 512, 8, 128), (16, 768, 3, 20), (129, 1024, 8, 128), (300, 4096, 16, 128),
                                        (2048, 14336, 8, 128), (40, 256, 0, 1)])
def test_rotate_group256(B, T, in_f, K, P):
    seed = synth.layer_seed(12, T + K)
    pairs, theta, alpha = synth.rotation_params(in_f, max(K, 1), seed, pairs_per_group=P, group=G256)
    if K == 0:
        pairs, theta = pairs[:0], theta[:0]
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G256)
    got = host(B.paro_rotate(rot, dev(x)))
    rows = np.arange(T) if T * in_f <= 4_000_000 else np.unique(
        np.concatenate([[0, T - 1], np.random.default_rng(T).choice(T, 64, replace=False)]))
    check_rotation(got[rows], x[rows], pairs, theta, alpha, group=G256)
    assert B.paro_fault_status() == 0


def test_rotate_group256_needs_multiple_of_256(B):
    pairs, theta, alpha = synth.rotation_params(384, 1, 3, pairs_per_group=64)
    with pytest.raises(B.ParoError):
        B.paro_rot_create(pairs[:, :1], theta[:, :1], alpha, group=G256)


@pytest.mark.parametrize("out_f,in_f", [(48, 512), (1024, 4096)])
def test_pack_dequant_group256_bit_exact(B, out_f, in_f):
    q, s, z = synth.w4_codes(out_f, in_f, seed=out_f + in_f, group=G256)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z), group=G256)
    got = host(B.paro_dequant(qw, sp, zp, in_f, out_f, group=G256))
    assert np.array_equal(got.view(np.uint16), O.dequantize(q, s, z, group=G256).view(np.uint16))


@pytest.mark.parametrize("out_f,in_f,K,P", [(64, 512, 8, 128), (32, 768, 4, 30)])
def test_quantize_group256_matches_oracle(B, out_f, in_f, K, P):
    seed = synth.layer_seed(12, out_f + K)
    pairs, theta, alpha = synth.rotation_params(in_f, K, seed, pairs_per_group=P, group=G256)
    w = synth.weight(out_f, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G256)
    q, s, z = (host(t) for t in B.paro_quantize_weights(rot, dev(w)))
    q0, s0, z0, _ = O.quantize_layer(w, pairs, theta, alpha, group=G256)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    assert np.array_equal(z, z0)
    assert np.array_equal(q, q0)


@pytest.mark.parametrize("T,in_f,out_f", [
    (1, 512, 512), (5, 768, 48), (16, 4096, 6144),          # decode kernel (tensor-core rotation first)
    (17, 512, 96), (300, 1024, 160), (2500, 512, 96),       # tensor-core GEMM
])
def test_linear_group256(B, T, in_f, out_f):
    seed = synth.layer_seed(12, T * 7 + in_f)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=128, group=G256)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G256)
    if out_f * in_f <= 1 << 20:
        w = synth.weight(out_f, in_f, seed)
        q, s, z, _ = O.quantize_layer(w, pairs, theta, alpha, group=G256)
    else:
        q, s, z = synth.w4_codes(out_f, in_f, seed, group=G256)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z), group=G256)
    x = synth.activations(T, in_f, seed)
    y = host(B.paro_linear_ex(rot, dev(x), qw, sp, zp, out_f, group=G256))
    rows = np.arange(out_f) if out_f <= 1040 else np.unique(
        np.concatenate([[0, out_f - 1], np.random.default_rng(seed).choice(out_f, 256, replace=False)]))
    toks = np.arange(T) if T <= 300 else np.unique(
        np.concatenate([[0, T - 1], np.random.default_rng(seed).choice(T, 40, replace=False)]))
    check_linear(y[np.ix_(toks, rows)], x[toks], pairs, theta, alpha, q[rows], s[rows], z[rows], group=G256)
    assert B.paro_fault_status() == 0
