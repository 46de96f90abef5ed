"""Groups of 64 channels (the speed end of the group-size knob, CSDN article,
section 5.2): rotation pairs inside 64-channel groups and W4G64 weights,
through the C ABI, against the fp64 oracle run with group = 64. Same bars as
test_gpu_parity.py (bit-exact codes and dequantisation; rotation and layer
tolerances from tests/parity.py)."""
import numpy as np
import pytest
import torch

import synth
from oracle import paro_oracle as O
from parity import check_linear, check_rotation

pytestmark = pytest.mark.gpu
G64 = 64


@pytest.fixture(scope="module")
def B(cuda_lib):
    from rotated_w4_linear_b200 import binding
    return binding


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("T,in_f,K,P", [(5, 512, 8, 32), (16, 384, 3, 7), (300, 4096, 8, 32), (40, 256, 0, 1)])
def test_rotate_group64(B, T, in_f, K, P):
    """Givens kernel (up to 16 tokens) and tensor-core kernel (above)."""
    seed = synth.layer_seed(10, T + K)
    pairs, theta, alpha = synth.rotation_params(in_f, max(K, 1), seed, pairs_per_group=P, group=G64)
    if K == 0:
        pairs, theta = pairs[:0], theta[:0]
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G64)
    check_rotation(host(B.paro_rotate(rot, dev(x))), x, pairs, theta, alpha, group=G64)
    assert B.paro_fault_status() == 0


def test_rotate_group64_pair_must_stay_in_its_group(B):
    pairs, theta, alpha = synth.rotation_params(256, 2, 3, pairs_per_group=32, group=G64)
    bad = pairs.copy()
    bad[0, 1, 0, 1] = 64                     # index outside a 64-channel group
    with pytest.raises(B.ParoError):
        B.paro_rot_create(bad, theta, alpha, group=G64)


@pytest.mark.parametrize("out_f,in_f", [(48, 384), (4096, 4096)])
def test_pack_dequant_group64_bit_exact(B, out_f, in_f):
    q, s, z = synth.w4_codes(out_f, in_f, seed=out_f + in_f, group=G64)
    for src in ((dev(q), dev(s), dev(z)), (torch.from_numpy(q), torch.from_numpy(s), torch.from_numpy(z))):
        qw, sp, zp = B.paro_pack_weights(*src, group=G64)
        got = host(B.paro_dequant(qw, sp, zp, in_f, out_f, group=G64))
        assert np.array_equal(got.view(np.uint16), O.dequantize(q, s, z, group=G64).view(np.uint16))


@pytest.mark.parametrize("out_f,in_f,K,P", [(64, 512, 8, 32), (32, 384, 4, 7)])
def test_quantize_group64_matches_oracle(B, out_f, in_f, K, P):
    seed = synth.layer_seed(10, out_f + K)
    pairs, theta, alpha = synth.rotation_params(in_f, K, seed, pairs_per_group=P, group=G64)
    w = synth.weight(out_f, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G64)
    q, s, z = (host(t) for t in B.paro_quantize_weights(rot, dev(w)))
    q0, s0, z0, _ = O.quantize_layer(w, pairs, theta, alpha, group=G64)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    assert np.array_equal(z, z0)
    assert np.array_equal(q, q0)


@pytest.mark.parametrize("T,in_f,out_f", [
    (1, 512, 512), (5, 384, 48), (16, 640, 1040), (12, 4096, 6144),    # decode kernel
    (17, 512, 96), (300, 256, 160), (2500, 384, 96),                   # tensor-core GEMM
])
def test_linear_group64(B, T, in_f, out_f):
    seed = synth.layer_seed(10, T * 7 + in_f)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=32, group=G64)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G64)
    if out_f * in_f <= 1 << 20:
        w = synth.weight(out_f, in_f, seed)
        q, s, z, _ = O.quantize_layer(w, pairs, theta, alpha, group=G64)
    else:
        q, s, z = synth.w4_codes(out_f, in_f, seed, group=G64)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z), group=G64)
    x = synth.activations(T, in_f, seed)
    y = host(B.paro_linear_ex(rot, dev(x), qw, sp, zp, out_f, group=G64))
    rows = np.arange(out_f) if out_f <= 1040 else np.unique(
        np.concatenate([[0, out_f - 1], np.random.default_rng(seed).choice(out_f, 256, replace=False)]))
    toks = np.arange(T) if T <= 300 else np.unique(
        np.concatenate([[0, T - 1], np.random.default_rng(seed).choice(T, 40, replace=False)]))
    check_linear(y[np.ix_(toks, rows)], x[toks], pairs, theta, alpha, q[rows], s[rows], z[rows], group=G64)
    assert B.paro_fault_status() == 0


def test_linear_group_mismatch_rejected(B):
    pairs, theta, alpha = synth.rotation_params(256, 2, 4, pairs_per_group=32, group=G64)
    rot = B.paro_rot_create(pairs, theta, alpha, group=G64)
    q, s, z = synth.w4_codes(32, 256, 4)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    with pytest.raises(B.ParoError):
        B.paro_linear_ex(rot, dev(synth.activations(4, 256, 4)), qw, sp, zp, 32, group=128)
