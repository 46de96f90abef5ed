"""Parity of the CUDA path (through the C ABI) with the CPU fp64 oracle.

Tolerances (stated for this layer, with the readings of the open points):
  * int4 unpack/dequant: bit-exact fp16;
  * offline quantiser: bit-exact q, s, z;
  * rotated activations: per-element relative error <= 1e-3 against fp64,
    the denominator floored at 1% of the element's group maximum (the
    literal, unfloored maximum is recorded beside it);
  * layer output: ||Y - Y_ref|| / ||Y_ref|| <= 2e-3, and per element
    |Y - Y_ref| <= max(1e-2, f + 2e-3), where f = |Y_x16 - Y_ref| +
    spacing16/2 is that element's error in the ideal fp16 pipeline (X'
    rounded to fp16, exact contraction, Y rounded to nearest fp16: Y_x16 is
    its value before the output rounding, spacing16 the fp16 spacing at the
    larger of |Y| and |Y_ref|) and 2e-3 the budget for fp32 accumulation and
    for X' elements that round to the other fp16 neighbour. An element may
    pass above 1e-2 only where the format itself forces it, and a result
    rounded to the wrong fp16 neighbour passes only within that budget of a
    rounding midpoint (tests/test_parity_bounds.py). The literal max |Y - Y_ref| and the pipeline's own maximum
    (the format floor) are recorded for every call.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import paro_oracle as O
from parity import check_linear, check_rotation

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda_lib):
    from rotated_w4_linear_b200 import binding
    return binding


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


# ---------------------------------------------------------------- rotation
@pytest.mark.parametrize("T,in_f,K,P", [
    (16, 512, 8, 64),      # the tiny single layer
    (1, 4096, 8, 64),
    (3, 4096, 1, 64),
    (17, 4096, 4, 64),
    (256, 4096, 8, 13),    # partial matchings: 13 of 64 pairs per group
    (9, 384, 8, 64),       # ragged token tile, odd group count
    (5, 256, 0, 1),        # K = 0: channel scaling only
])
def test_rotate_parity(B, T, in_f, K, P):
    seed = synth.layer_seed(1, T + K)
    pairs, theta, alpha = synth.rotation_params(in_f, max(K, 1), seed, pairs_per_group=P)
    if K == 0:
        pairs, theta = pairs[:0], theta[:0]
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    got = host(B.paro_rotate(rot, dev(x)))
    check_rotation(got, x, pairs, theta, alpha)


@pytest.mark.parametrize("in_f,K,P", [(4096, 8, 64), (14336, 16, 13), (384, 3, 64)])
def test_rotate_givens_rows_do_not_depend_on_the_batch(B, in_f, K, P):
    """Batches of at most 16 tokens take the Givens quad kernel (float4
    exchange, packed f32x2 arithmetic; from 9 tokens on with each layer's
    tables loaded during the layer before). The operations on a row and
    their order are the same in every batch size: identical bits."""
    seed = synth.layer_seed(1, 77 + K)
    pairs, theta, alpha = synth.rotation_params(in_f, K, seed, pairs_per_group=P)
    x = synth.activations(16, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    big = host(B.paro_rotate(rot, dev(x)))
    for T in (1, 7, 8, 9, 12):
        small = host(B.paro_rotate(rot, dev(x[16 - T:])))
        assert np.array_equal(small.view(np.uint16), big[16 - T:].view(np.uint16)), T
    check_rotation(big, x, pairs, theta, alpha)


@pytest.mark.parametrize("T,in_f,K,P", [
    (17, 4096, 8, 64),      # the smallest batch the tensor cores take
    (64, 640, 2, 64),
    (128, 384, 8, 64),      # one 128-token tile, three groups
    (129, 4096, 8, 64),     # ragged second tile
    (300, 256, 1, 64),      # one layer: a sparse M
    (300, 384, 4, 13),      # partial matchings
    (1000, 4096, 16, 64),   # sixteen layers
    (777, 640, 0, 1),       # K = 0: M = diag(1/alpha)
    (2048, 14336, 8, 64),   # down-projection width: 112 groups
])
def test_rotate_tensor_core_parity(B, T, in_f, K, P):
    """Above 16 tokens, each group's diag(1/alpha) R_1^T .. R_K^T is applied
    as one dense matrix on the tensor cores (fp16 hi + lo parts, fp32
    accumulation): every element against the fp64 oracle."""
    seed = synth.layer_seed(1, 500 + T + K)
    pairs, theta, alpha = synth.rotation_params(in_f, max(K, 1), seed, pairs_per_group=P)
    if K == 0:
        pairs, theta = pairs[:0], theta[:0]
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    got = host(B.paro_rotate(rot, dev(x)))
    if T * in_f > 4_000_000:                           # large: sampled rows, first and last included
        rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(T).choice(T, 96, replace=False)]))
        check_rotation(got[rows], x[rows], pairs, theta, alpha)
    else:
        check_rotation(got, x, pairs, theta, alpha)
    assert B.paro_fault_status() == 0
    # a row's result does not depend on the batch or the tile it is in
    twice = host(B.paro_rotate(rot, dev(np.concatenate([x[T // 3:], x]))))
    assert np.array_equal(twice[T - T // 3:].view(np.uint16), got.view(np.uint16))


@pytest.mark.parametrize("T", [2048, 8192])
def test_rotate_full_size_sampled_rows(B, T):
    seed = synth.layer_seed(1, T)
    pairs, theta, alpha = synth.rotation_params(4096, 8, seed)
    x = synth.activations(T, 4096, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    got = host(B.paro_rotate(rot, dev(x)))
    rows = np.random.default_rng(T).choice(T, 64, replace=False)
    rows[0], rows[-1] = 0, T - 1
    check_rotation(got[rows], x[rows], pairs, theta, alpha)


def test_rotate_empty_and_invalid(B):
    pairs, theta, alpha = synth.rotation_params(256, 2, 1)
    rot = B.paro_rot_create(pairs, theta, alpha)
    x = torch.empty((0, 256), dtype=torch.float16, device="cuda")
    assert B.paro_rotate(rot, x).shape == (0, 256)
    bad = pairs.copy()
    bad[1, 0, 3, 1] = bad[1, 0, 2, 0]
    with pytest.raises(B.ParoError):
        B.paro_rot_create(bad, theta, alpha)
    with pytest.raises(B.ParoError):
        B.paro_rot_create(pairs, theta, np.zeros_like(alpha))


# ---------------------------------------------------------------- int4 format
@pytest.mark.parametrize("out_f,in_f", [(48, 384), (6144, 4096), (4096, 14336)])
def test_pack_dequant_bit_exact(B, out_f, in_f):
    q, s, z = synth.w4_codes(out_f, in_f, seed=out_f + in_f)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    got = host(B.paro_dequant(qw, sp, zp, in_f, out_f))
    ref = O.dequantize(q, s, z)
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


def test_dequant_all_codes_and_extreme_scales(B):
    # every (q, z) pair, scales spanning the fp16 normal range
    out_f, in_f = 16, 256 * 2
    q = np.tile(np.arange(16, dtype=np.uint8), (out_f, in_f // 16))
    z = (np.arange(out_f * 4).reshape(out_f, 4) % 16).astype(np.uint8)
    s = np.array([[2.0 ** -14, 0.000123, 0.75, 4095.0]] * out_f, np.float16)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    got = host(B.paro_dequant(qw, sp, zp, in_f, out_f))
    assert np.array_equal(got.view(np.uint16), O.dequantize(q, s, z).view(np.uint16))


# ---------------------------------------------------------------- converter
@pytest.mark.parametrize("out_f,in_f,K,P", [(64, 512, 8, 64), (256, 4096, 8, 64), (32, 384, 4, 13)])
def test_quantize_matches_oracle(B, out_f, in_f, K, P):
    seed = synth.layer_seed(0, out_f + K)
    pairs, theta, alpha = synth.rotation_params(in_f, K, seed, pairs_per_group=P)
    w = synth.weight(out_f, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    q, s, z = (host(t) for t in B.paro_quantize_weights(rot, dev(w)))
    q0, s0, z0, _ = O.quantize_layer(w, pairs, theta, alpha)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    assert np.array_equal(z, z0)
    assert np.array_equal(q, q0)


# ---------------------------------------------------------------- the layer
def _layer(B, in_f, out_f, K, P, seed, oracle_quant=True):
    pairs, theta, alpha = synth.rotation_params(in_f, K, seed, pairs_per_group=P)
    if oracle_quant:
        w = synth.weight(out_f, in_f, seed)
        q, s, z, _ = O.quantize_layer(w, pairs, theta, alpha)
    else:
        q, s, z = synth.w4_codes(out_f, in_f, seed)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    return (pairs, theta, alpha, q, s, z), (qw, sp, zp)


@pytest.mark.parametrize("T,in_f,out_f,K,P", [
    (16, 512, 512, 8, 64),     # the tiny single layer, every output
    (1, 512, 512, 8, 64),
    (3, 384, 48, 8, 64),
    (8, 256, 80, 4, 13),
    (9, 384, 48, 1, 64),
    (16, 128, 272, 2, 64),     # one group (half a 256-channel stage), ragged 128-row tile
    (12, 640, 1040, 8, 64),    # odd stage count, many tiles split over CTAs
    (17, 512, 96, 8, 64),      # > 16 tokens: prefill path (tensor-core GEMM)
    (40, 384, 48, 8, 64),      # partial 128-row tile, odd group count
    (130, 512, 256, 8, 64),    # two 128-token tiles, ragged
    (300, 256, 160, 4, 13),    # 256-token tiles, ragged rows and tokens
    (2500, 384, 96, 8, 64),    # twenty 128-token tiles, ragged last tile
])
def test_linear_parity_exhaustive(B, T, in_f, out_f, K, P):
    seed = synth.layer_seed(0, T * 7 + K)
    (pairs, theta, alpha, q, s, z), (qw, sp, zp) = _layer(B, in_f, out_f, K, P, seed)
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    ws = B.workspace(T, in_f, out_f)
    ws.fill_(0xA5)                     # scratch: any initial content
    for _ in range(2):
        y = host(B.paro_linear(rot, dev(x), qw, sp, zp, out_f, ws=ws))
        check_linear(y, x, pairs, theta, alpha, q, s, z)
    assert B.paro_fault_status() == 0


@pytest.mark.parametrize("T,in_f,out_f", [(1, 512, 96), (16, 384, 272), (40, 512, 160), (300, 256, 48)])
def test_linear_bias(B, T, in_f, out_f):
    """Y = (X T^-1) w_hat^T + b on the decode (T <= 16) and prefill paths."""
    seed = synth.layer_seed(5, T + in_f)
    (pairs, theta, alpha, q, s, z), (qw, sp, zp) = _layer(B, in_f, out_f, 8, 64, seed)
    x = synth.activations(T, in_f, seed)
    b = (np.random.default_rng(seed).standard_normal(out_f) * 4).astype(np.float16)
    rot = B.paro_rot_create(pairs, theta, alpha)
    y = host(B.paro_linear_bias(rot, dev(x), qw, sp, zp, dev(b), out_f))
    check_linear(y, x, pairs, theta, alpha, q, s, z, bias=b)
    y0 = host(B.paro_linear_bias(rot, dev(x), qw, sp, zp, None, out_f))       # null bias = paro_linear
    assert np.array_equal(y0.view(np.uint16), host(B.paro_linear(rot, dev(x), qw, sp, zp, out_f)).view(np.uint16))


@pytest.mark.parametrize("T", [1, 5, 16])
def test_linear_unrotated(B, T):
    in_f, out_f = 512, 128
    q, s, z = synth.w4_codes(out_f, in_f, seed=T)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    x = synth.activations(T, in_f, seed=T)
    y = host(B.paro_linear(None, dev(x), qw, sp, zp, out_f))
    check_linear(y, x, None, None, None, q, s, z)


LLAMA = [(4096, 6144), (4096, 4096), (4096, 28672), (14336, 4096)]


@pytest.mark.parametrize("T", [1, 4, 16])
@pytest.mark.parametrize("in_f,out_f", LLAMA)
def test_linear_decode_full_size_sampled(B, T, in_f, out_f):
    seed = synth.layer_seed(2, in_f + out_f + T)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
    q, s, z = synth.w4_codes(out_f, in_f, seed)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    y = host(B.paro_linear(rot, dev(x), qw, sp, zp, out_f))
    rows = np.random.default_rng(seed).choice(out_f, 256, replace=False)
    rows[0], rows[-1] = 0, out_f - 1
    check_linear(y[:, rows], x, pairs, theta, alpha, q[rows], s[rows], z[rows])


def _random_shapes(n, seed):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        yield (int(rng.integers(1, 17)), 128 * int(rng.integers(1, 97)), 16 * int(rng.integers(1, 769)))


@pytest.mark.parametrize("T,in_f,out_f", list(_random_shapes(12, 2024)))
def test_linear_decode_random_shapes_sampled(B, T, in_f, out_f):
    """The decode planner's tilings (k-chunk, cluster size, row tile, token
    tiles) on random shapes up to 12288 inputs and 12288 outputs."""
    seed = synth.layer_seed(6, T + in_f + out_f)
    pairs, theta, alpha = synth.rotation_params(in_f, 4, seed, pairs_per_group=48)
    q, s, z = synth.w4_codes(out_f, in_f, seed)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    y = host(B.paro_linear(rot, dev(x), qw, sp, zp, out_f))
    rows = np.unique(np.concatenate([[0, out_f - 1], np.random.default_rng(seed).choice(out_f, min(out_f, 96), replace=False)]))
    check_linear(y[:, rows], x, pairs, theta, alpha, q[rows], s[rows], z[rows])
    assert B.paro_fault_status() == 0


# Qwen3-shaped decoder-layer linears: 4B-like (hidden 2560, intermediate 9728,
# 32 q / 8 kv heads x 128) and 14B-like (hidden 5120, intermediate 17408,
# 40 q / 8 kv heads x 128); QKV and gate+up fused.
QWEN3 = [(2560, 6144), (4096, 2560), (2560, 19456), (9728, 2560),
         (5120, 7168), (5120, 5120), (5120, 34816), (17408, 5120)]


@pytest.mark.parametrize("T", [1, 8])
@pytest.mark.parametrize("in_f,out_f", QWEN3)
def test_linear_decode_qwen3_shapes_sampled(B, T, in_f, out_f):
    seed = synth.layer_seed(4, in_f + out_f + T)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
    q, s, z = synth.w4_codes(out_f, in_f, seed)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    y = host(B.paro_linear(rot, dev(x), qw, sp, zp, out_f))
    rows = np.random.default_rng(seed).choice(out_f, 128, replace=False)
    rows[0], rows[-1] = 0, out_f - 1
    check_linear(y[:, rows], x, pairs, theta, alpha, q[rows], s[rows], z[rows])


def _prefill_sampled(B, T, in_f, out_f, seed, n_tok=16, n_rows=128):
    """One full-size prefill call; the oracle checks n_tok sampled tokens
    (first and last included) over n_rows sampled output rows (first and
    last included)."""
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
    q, s, z = synth.w4_codes(out_f, in_f, seed)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    y = B.paro_linear(rot, dev(x), qw, sp, zp, out_f)
    rng = np.random.default_rng(seed)
    toks = rng.choice(T, n_tok, replace=False)
    toks[0], toks[-1] = 0, T - 1
    rows = rng.choice(out_f, n_rows, replace=False)
    rows[0], rows[-1] = 0, out_f - 1
    ys = host(y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(rows).cuda()])
    del y
    check_linear(ys, x[toks], pairs, theta, alpha, q[rows], s[rows], z[rows])
    assert B.paro_fault_status() == 0


@pytest.mark.parametrize("in_f,out_f", QWEN3)
def test_linear_prefill_qwen3_shapes_sampled(B, in_f, out_f):
    _prefill_sampled(B, 4096, in_f, out_f, synth.layer_seed(4, in_f + out_f))


@pytest.mark.parametrize("T", [2048, 8192])
@pytest.mark.parametrize("in_f,out_f", LLAMA)
def test_linear_prefill_full_size_sampled(B, T, in_f, out_f):
    _prefill_sampled(B, T, in_f, out_f, synth.layer_seed(3, in_f + out_f + T), n_tok=24, n_rows=256)


@pytest.mark.parametrize("T", [5, 300])
def test_oneshot_calls_and_host_packing(B, T):
    """paro_rotate_once / paro_linear_once (the rotation given as pairs,
    theta, alpha) give the handle calls' bits; packing from host tensors
    gives the device packing's bytes."""
    in_f, out_f = 512, 96
    seed = synth.layer_seed(7, T)
    (pairs, theta, alpha, q, s, z), (qw, sp, zp) = _layer(B, in_f, out_f, 8, 64, seed)
    qh, sh, zh = (B.paro_pack_weights(torch.from_numpy(q), torch.from_numpy(s), torch.from_numpy(z)))
    for a, b in ((qw, qh), (sp, sh), (zp, zh)):
        assert torch.equal(a, b)
    x = synth.activations(T, in_f, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    xr = host(B.paro_rotate(rot, dev(x)))
    xr1 = host(B.paro_rotate_once(dev(x), pairs, theta, alpha))
    assert np.array_equal(xr.view(np.uint16), xr1.view(np.uint16))
    y = host(B.paro_linear(rot, dev(x), qw, sp, zp, out_f))
    y1 = host(B.paro_linear_once(dev(x), pairs, theta, alpha, qh, sh, zh, out_f))
    assert np.array_equal(y.view(np.uint16), y1.view(np.uint16))
    check_linear(y1, x, pairs, theta, alpha, q, s, z)


def test_bounded_wait_runs_out_and_the_context_survives(B):
    """Failure detection without a GPU fault: a kernel waits, with a 1 ms
    limit, on an mbarrier at which nothing arrives; the wait gives up, the
    kernel returns, the fault word holds code 6 until cleared, and the next
    layer call on the same context is correct."""
    B.paro_fault_status(clear=True)
    B.paro_check_wait_timeout(1000)
    torch.cuda.synchronize()
    assert B.paro_fault_status() == 6
    assert B.paro_fault_status(clear=True) == 6
    assert B.paro_fault_status() == 0
    seed = synth.layer_seed(8, 1)
    (pairs, theta, alpha, q, s, z), (qw, sp, zp) = _layer(B, 384, 48, 8, 64, seed)
    x = synth.activations(40, 384, seed)
    rot = B.paro_rot_create(pairs, theta, alpha)
    check_linear(host(B.paro_linear(rot, dev(x), qw, sp, zp, 48)), x, pairs, theta, alpha, q, s, z)
    assert B.paro_fault_status() == 0


def test_prefill_graph_replays_keep_the_fault_word_clear(B):
    """The prefill path (tensor-core rotation, then the GEMM as a programmatic
    dependent launch) replayed back to back from a CUDA graph: no bounded
    wait runs out, and every replay gives the first replay's bits."""
    T, shapes = 2048, [(4096, 6144), (14336, 1024), (4096, 4096)]
    calls = []
    for i, (in_f, out_f) in enumerate(shapes):
        seed = synth.layer_seed(13, i)
        pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
        q, s, z = synth.w4_codes(out_f, in_f, seed)
        qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
        calls.append(dict(rot=B.paro_rot_create(pairs, theta, alpha), x=dev(synth.activations(T, in_f, seed)),
                          qw=qw, sp=sp, zp=zp, out=out_f, y=torch.empty((T, out_f), dtype=torch.float16, device="cuda"),
                          ws=B.workspace(T, in_f, out_f)))

    def step():
        for c in calls:
            B.paro_linear(c["rot"], c["x"], c["qw"], c["sp"], c["zp"], c["out"], Y=c["y"], ws=c["ws"])

    B.paro_fault_status(clear=True)
    step()
    torch.cuda.synchronize()
    first = [c["y"].clone() for c in calls]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(60):
        g.replay()
    torch.cuda.synchronize()
    assert B.paro_fault_status() == 0
    for c, y0 in zip(calls, first):
        assert torch.equal(c["y"], y0)
    del g



def test_decode_calls_of_several_shapes_share_one_workspace(B):
    """Decode calls whose grids differ in size, one after another on one
    workspace (eager, then 40 replays of a CUDA graph of them, each rotation
    a programmatic dependent of the decode kernel before it): no wait runs
    out, and every output matches the oracle."""
    T = 16
    shapes = [(4096, 6144), (4096, 4096), (4096, 28672), (14336, 4096), (640, 272)]
    calls = []
    for i, (in_f, out_f) in enumerate(shapes):
        seed = synth.layer_seed(15, i)
        pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
        q, s, z = synth.w4_codes(out_f, in_f, seed)
        qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z))
        x = synth.activations(T, in_f, seed)
        calls.append(dict(p=(pairs, theta, alpha, q, s, z), x=x, xd=dev(x), rot=B.paro_rot_create(pairs, theta, alpha),
                          qw=qw, sp=sp, zp=zp, out=out_f,
                          y=torch.empty((T, out_f), dtype=torch.float16, device="cuda")))
    ws = B.workspace(T, max(i for i, _ in shapes), max(o for _, o in shapes))

    def step():
        for c in calls:
            B.paro_linear(c["rot"], c["xd"], c["qw"], c["sp"], c["zp"], c["out"], Y=c["y"], ws=ws)

    def check():
        for c in calls:
            pairs, theta, alpha, q, s, z = c["p"]
            rows = np.random.default_rng(c["out"]).choice(c["out"], min(c["out"], 96), replace=False)
            check_linear(host(c["y"])[:, rows], c["x"], pairs, theta, alpha, q[rows], s[rows], z[rows])

    B.paro_fault_status(clear=True)
    step()
    torch.cuda.synchronize()
    check()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for c in calls:
        c["y"].zero_()
    for _ in range(40):
        g.replay()
    torch.cuda.synchronize()
    assert B.paro_fault_status() == 0
    check()
    del g


@pytest.mark.parametrize("group", [128, 64])
def test_prepared_layer_matches_the_oracle(B, group):
    """ParoLinear (weights, bias and workspace checked once, the workspace
    grown with the batch) over decode and prefill batches, against the
    oracle; a wrongly shaped X is refused before any launch."""
    in_f, out_f = 640, 272
    seed = synth.layer_seed(16, group)
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed, pairs_per_group=group // 2, group=group)
    q, s, z = synth.w4_codes(out_f, in_f, seed, group=group)
    qw, sp, zp = B.paro_pack_weights(dev(q), dev(s), dev(z), group=group)
    b = (np.random.default_rng(seed).standard_normal(out_f) * 2).astype(np.float16)
    rot = B.paro_rot_create(pairs, theta, alpha, group=group)
    layer = B.ParoLinear(rot, qw, sp, zp, in_f, out_f, group=group, bias=dev(b))
    for T in (1, 16, 5, 300):
        x = synth.activations(T, in_f, seed + T)
        y = torch.empty((T, out_f), dtype=torch.float16, device="cuda")
        layer(dev(x), Y=y)
        check_linear(host(y), x, pairs, theta, alpha, q, s, z, bias=b, group=group)
    with pytest.raises(TypeError):
        layer(torch.zeros((4, in_f + 128), dtype=torch.float16, device="cuda"))
    with pytest.raises(TypeError):
        layer(torch.zeros((4, in_f), dtype=torch.float32, device="cuda"))
    assert B.paro_fault_status() == 0
