"""Pins for the CPU oracle against facts the pages and the mathematics fix.

None of these compares the oracle with itself: each check uses a hand-worked
value, a closed form, an independent library routine (numpy.linalg.inv) or a
brute-force loop.
"""
import os

import numpy as np
import pytest

import synth
from oracle import paro_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---- 2x2 closed form (CSDN article, section 2.2 matrix) --------------------
def test_givens_2x2_golden():
    for c, s, vi, vj, ei, ej in (map(float, r) for r in _rows("givens_2x2.txt")):
        th = np.float32(np.arctan2(s, c))
        pairs = np.array([[[0, 1]]], dtype=np.int16)          # one group of 2
        out = O.givens_layer(np.array([[vi, vj]]), pairs, np.array([[th]]), group=2)
        assert np.allclose(out[0], [ei, ej], atol=2e-7), (c, s, vi, vj, out)


def test_swapping_pair_order_negates_angle():
    v = np.array([[0.3, -1.7]])
    th = np.float32(0.9)
    a = O.givens_layer(v, np.array([[[0, 1]]], np.int16), np.array([[th]]), group=2)
    b = O.givens_layer(v, np.array([[[1, 0]]], np.int16), np.array([[-th]]), group=2)
    assert np.allclose(a, b, atol=1e-15)


def test_rotate_two_layers_golden():
    rows = {r[0]: r[1:] for r in _rows("rotate_k2.txt") if r[0] in ("x", "alpha", "expect")}
    layers = [r[1:] for r in _rows("rotate_k2.txt") if r[0] == "layer"]
    layers2 = [r[1:] for r in _rows("rotate_k2.txt") if r[0] == "layer2"]
    x = np.array([list(map(float, rows["x"]))])
    alpha = np.array(list(map(float, rows["alpha"])), np.float32)
    pairs = np.zeros((2, 1, 2, 2), np.int16)
    theta = np.zeros((2, 1, 2), np.float32)
    for t, lay in enumerate((layers, layers2)):
        for p, (i, j, c, s) in enumerate(lay):
            pairs[t, 0, p] = (int(i), int(j))
            theta[t, 0, p] = np.arctan2(float(s), float(c))
    got = O.rotate_activations(x, pairs, theta, alpha, group=4)
    assert np.allclose(got[0], list(map(float, rows["expect"])), atol=2e-6), got


# ---- structure: orthogonality, inverse, dense brute force -------------------
def _small(seed, in_f=16, K=3, group=8, P=None):
    P = P or group // 2
    pairs = synth.matchings(in_f, K, seed, pairs_per_group=P, group=group)
    theta = synth.angles(K, in_f // group, P, seed)
    alpha = synth.channel_scales(in_f, seed)
    return pairs, theta, alpha


def test_norm_preserved_when_alpha_is_one():
    pairs, theta, _ = synth.rotation_params(512, 8, seed=3)
    x = synth.activations(7, 512, seed=3).astype(np.float64)
    xr = O.rotate_activations(x, pairs, theta, np.ones(512, np.float32))
    n0 = np.linalg.norm(x.reshape(7, 4, 128), axis=2)
    n1 = np.linalg.norm(xr.reshape(7, 4, 128), axis=2)
    assert np.allclose(n0, n1, rtol=1e-13)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_pairwise_matches_dense_bruteforce(seed):
    group = 8
    pairs, theta, alpha = _small(seed, group=group)
    T = O.dense_transform(pairs, theta, alpha, group=group)
    w = np.random.default_rng(seed).standard_normal((5, 16))
    x = np.random.default_rng(seed + 10).standard_normal((3, 16))
    # weight side: every row w[o] (input-channel axis) maps to T w[o]
    assert np.allclose(O.transform_weight(w, pairs, theta, alpha, group), w @ T.T, atol=1e-14)
    # activation side: X T^-1 with an independent inverse
    assert np.allclose(O.rotate_activations(x, pairs, theta, alpha, group), x @ np.linalg.inv(T), atol=1e-12)
    # T^-1 T = I, and R_K..R_1 is orthogonal
    R = T @ np.diag(1.0 / alpha.astype(np.float64))
    assert np.allclose(R @ R.T, np.eye(16), atol=1e-14)
    assert np.isclose(np.linalg.det(R), 1.0)


def test_dense_single_pair_is_page_matrix():
    pairs = np.array([[[[1, 0]]]], np.int16)     # pair (i=1, j=0)
    theta = np.array([[[0.7]]], np.float32)
    T = O.dense_transform(pairs, theta, np.ones(2, np.float32), group=2)
    c, s = np.cos(np.float64(np.float32(0.7))), np.sin(np.float64(np.float32(0.7)))
    # rows/cols in (i, j) order must be [[c, -s], [s, c]]
    assert np.allclose(T[np.ix_([1, 0], [1, 0])], [[c, -s], [s, c]], atol=1e-15)


def test_equivalence_before_quantisation():
    """(X T^-1)(T W) = X W (CSDN article, section 2.1)."""
    pairs, theta, alpha = synth.rotation_params(512, 8, seed=5)
    x = synth.activations(9, 512, seed=5).astype(np.float64)
    w = synth.weight(64, 512, seed=5).astype(np.float64)
    lhs = O.rotate_activations(x, pairs, theta, alpha) @ O.transform_weight(w, pairs, theta, alpha).T
    rhs = x @ w.T
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(rhs) < 1e-12


def test_layer_order_matters():
    pairs, theta, alpha = synth.rotation_params(256, 4, seed=8)
    x = synth.activations(4, 256, seed=8)
    a = O.rotate_activations(x, pairs, theta, alpha)
    b = O.rotate_activations(x, pairs[::-1].copy(), theta[::-1].copy(), alpha)
    assert np.max(np.abs(a - b)) > 1e-2


def test_partial_matching_leaves_unpaired_channels_scaled_only():
    pairs, theta, alpha = synth.rotation_params(256, 8, seed=9, pairs_per_group=13)
    x = synth.activations(5, 256, seed=9).astype(np.float64)
    xr = O.rotate_activations(x, pairs, theta, alpha)
    touched = np.zeros(256, bool)
    for g in range(2):
        touched[g * 128 + pairs[:, g].reshape(-1).astype(int)] = True
    assert touched.sum() < 256
    assert np.array_equal(xr[:, ~touched], x[:, ~touched] / alpha[~touched].astype(np.float64))


def test_zero_angles_unit_scales_is_identity():
    pairs, theta, _ = synth.rotation_params(256, 8, seed=2)
    x = synth.activations(3, 256, seed=2).astype(np.float64)
    xr = O.rotate_activations(x, pairs, np.zeros_like(theta), np.ones(256, np.float32))
    assert np.array_equal(xr, x)


def test_invalid_pairs_rejected():
    pairs, theta, alpha = synth.rotation_params(256, 2, seed=2)
    bad = pairs.copy()
    bad[0, 0, 1, 0] = bad[0, 0, 0, 0]            # channel used twice in one layer
    with pytest.raises(AssertionError):
        O.rotate_activations(np.zeros((1, 256)), bad, theta, alpha)
    bad = pairs.copy()
    bad[0, 1, 0, 1] = 128                        # index outside its group
    with pytest.raises(AssertionError):
        O.rotate_activations(np.zeros((1, 256)), bad, theta, alpha)


# ---- quantiser ----------------------------------------------------------------
def test_rtn_golden():
    rows = {r[0]: list(map(float, r[1:])) for r in _rows("rtn_example.txt")}
    q, s, z = O.rtn_quantize(np.array([rows["w"]]), group=4)
    assert float(s[0, 0]) == rows["s"][0]
    assert int(z[0, 0]) == int(rows["z"][0])
    assert q[0].tolist() == [int(v) for v in rows["q"]]
    wh = O.dequantize(q, s, z, group=4)
    assert wh.dtype == np.float16 and wh[0].astype(np.float64).tolist() == rows["w_hat"]


def test_rtn_invariants():
    w = synth.weight(32, 512, seed=4).astype(np.float64)
    q, s, z = O.rtn_quantize(w)
    assert q.max() <= 15 and z.max() <= 15
    sf = np.repeat(s.astype(np.float64), 128, axis=1)
    zf = np.repeat(z.astype(np.float64), 128, axis=1)
    exact = (q - zf) * sf
    unclipped = (q > 0) & (q < 15)
    assert np.all(np.abs(w - exact)[unclipped] <= sf[unclipped] / 2 * (1 + 1e-12))
    # clipping only at the group extremes, by at most one step plus the zero rounding
    assert np.all(np.abs(w - exact) <= sf * (1 + 1e-9))
    # w_hat is exactly the fp16 value nearest the exact product
    wh = O.dequantize(q, s, z).astype(np.float64)
    spacing = np.abs(np.spacing(exact.astype(np.float16))).astype(np.float64)
    assert np.all(np.abs(wh - exact) <= spacing / 2)


def test_rtn_degenerate_and_zero_groups():
    w = np.zeros((2, 128))
    w[1, :] = 0.0
    q, s, z = O.rtn_quantize(w)
    assert np.all(s.astype(np.float64) == 2.0 ** -14)
    assert np.all(q == 0) and np.all(z == 0)
    assert np.all(O.dequantize(q, s, z) == 0)


def test_dequant_exhaustive_codes():
    """Every (q, z) pair at several scales: fp16((q-z)*s) equals the fp16 value
    nearest the exact rational product, found by brute force over the fp16 grid."""
    grid = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)   # finite >= 0
    for s in (0.199951171875, 0.0123443603515625, 2.0 ** -14, 3.0517578125e-05 * 3, 1.5):
        qq, zz = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
        q = qq.reshape(1, -1).astype(np.uint8)
        # one "group" per (q, z): use group size 1 with per-element s and z
        got = O.dequantize(q, np.full((1, 256), s, np.float16), zz.reshape(1, -1).astype(np.uint8), group=1)
        sv = float(np.float16(s))
        for k in range(256):
            exact = (int(qq.flat[k]) - int(zz.flat[k])) * sv
            a = abs(exact)
            idx = np.searchsorted(grid, a)
            cands = [grid[i] for i in (idx - 1, idx) if 0 <= i < grid.size]
            best = min(cands, key=lambda g: (abs(g - a), int(np.float16(g).view(np.uint16)) & 1))
            assert float(got[0, k]) == np.copysign(best, exact) or (best == 0 and got[0, k] == 0)


# ---- the layer ------------------------------------------------------------------
def test_linear_plain_w4g128_bruteforce():
    """theta = 0, alpha = 1 reduces the layer to plain W4G128; compare with a
    scalar int4 GEMM loop."""
    pairs, theta, _ = synth.rotation_params(256, 2, seed=6)
    x = synth.activations(3, 256, seed=6)
    w = synth.weight(8, 256, seed=6)
    ones = np.ones(256, np.float32)
    q, s, z, _ = O.quantize_layer(w, pairs, np.zeros_like(theta), ones)
    y = O.linear(x, pairs, np.zeros_like(theta), ones, q, s, z)
    for t in range(3):
        for o in range(8):
            acc = 0.0
            for c in range(256):
                g = c // 128
                wh = float(np.float16((int(q[o, c]) - int(z[o, g])) * float(s[o, g])))
                acc += float(x[t, c]) * wh
            assert abs(acc - y[t, o]) <= 1e-12 * max(1.0, abs(acc))


def test_linear_is_rotated_times_dequantised():
    pairs, theta, alpha = synth.rotation_params(512, 8, seed=7)
    x = synth.activations(4, 512, seed=7)
    w = synth.weight(16, 512, seed=7)
    q, s, z, wt = O.quantize_layer(w, pairs, theta, alpha)
    y = O.linear(x, pairs, theta, alpha, q, s, z)
    # distance to the unquantised rotated layer is bounded by the weight error
    xr = O.rotate_activations(x, pairs, theta, alpha)
    y0 = xr @ wt.T
    wh = O.dequantize(q, s, z).astype(np.float64)
    for t in range(4):
        assert np.linalg.norm(y[t] - y0[t]) <= np.linalg.norm(xr[t]) * np.linalg.norm(wh - wt, 2) * (1 + 1e-9)
    # and the rotated weight is what was quantised
    assert np.allclose(O.dequantize(q, s, z).astype(np.float64), wt, atol=np.repeat(s.astype(np.float64), 128, 1).max())


def test_error_measures():
    ref = np.array([[1.0, -2.0, 0.0, 0.001] * 32])
    got = ref.copy()
    got[0, 0] += 1e-3
    fl, lit = O.rotation_rel_error(got, ref)
    assert np.isclose(fl, 1e-3) and np.isclose(lit, 1e-3)
    got = ref.copy()
    got[0, 3] += 1e-5                           # tiny element: floor at 1% of the group max 2.0
    fl, lit = O.rotation_rel_error(got, ref)
    assert np.isclose(fl, 1e-5 / 0.02) and np.isclose(lit, 1e-2)
    rel, mx = O.output_errors(np.array([3.0, 4.0]), np.array([3.0, 4.5]))
    assert np.isclose(mx, 0.5) and np.isclose(rel, 0.5 / np.hypot(3, 4.5))


def test_bias_is_added_once_per_output_column():
    """CSDN article, section 2.1: Y = XW + b. With zero codes at zero point
    0 and any scale (w_hat = 0) the layer returns exactly b on every row;
    for real codes, adding b shifts each column by b and nothing else."""
    rng = np.random.default_rng(7)
    T, in_f, out_f = 3, 256, 40
    pairs, theta, alpha = synth.rotation_params(in_f, 2, 11)
    x = synth.activations(T, in_f, 11)
    b = rng.standard_normal(out_f).astype(np.float16)
    q0 = np.zeros((out_f, in_f), np.uint8)
    z0 = np.zeros((out_f, in_f // 128), np.uint8)
    s0 = np.full((out_f, in_f // 128), 0.5, np.float16)
    y0 = O.linear(x, pairs, theta, alpha, q0, s0, z0, bias=b)
    assert np.array_equal(y0, np.broadcast_to(b.astype(np.float64), (T, out_f)))
    q, s, z = synth.w4_codes(out_f, in_f, 12)
    ya = O.linear(x, pairs, theta, alpha, q, s, z)
    yb = O.linear(x, pairs, theta, alpha, q, s, z, bias=b)
    bb = np.broadcast_to(b.astype(np.float64), (T, out_f))
    assert np.all(np.abs((yb - ya) - bb) <= 1e-12 * (np.abs(ya) + np.abs(bb)))


# ---- the ideal fp16 pipeline (format floor of the output tolerance) ------------
def _fp16_pipeline_layer():
    """The tiny layer of tests/golden/fp16_pipeline.txt: one group, one layer
    with pair (0, 1) at theta = 0, alpha = 3, two output rows."""
    pairs = np.zeros((1, 1, 1, 2), np.int16)
    pairs[0, 0, 0] = (0, 1)
    theta = np.zeros((1, 1, 1), np.float32)
    alpha = np.full(128, 3.0, np.float32)
    q = np.zeros((2, 128), np.uint8)
    q[0, :2] = 3
    q[1, :] = 1
    q[1, 0], q[1, 1] = 2, 0
    z = np.array([[0], [1]], np.uint8)
    s = np.ones((2, 1), np.float16)
    rows = {r[0]: [float(v) for v in r[1:]] for r in _rows("fp16_pipeline.txt")}
    x = np.zeros((2, 128), np.float16)
    x[0, :2], x[1, :2] = rows["x0"], rows["x1"]
    return (x, pairs, theta, alpha, q, s, z), rows


def test_fp16_pipeline_golden():
    """X' rounded to fp16, exact contraction, Y rounded to fp16 (or not), with
    and without a bias: every value worked by hand, including three
    round-half-to-even ties."""
    layer, rows = _fp16_pipeline_layer()
    b = np.array(rows["bias"], np.float16)
    un = O.linear_fp16_pipeline(*layer, round_output=False)
    rd = O.linear_fp16_pipeline(*layer, round_output=True)
    assert un.dtype == np.float64 and rd.dtype == np.float16
    assert un.reshape(-1).tolist() == rows["unrounded"]
    assert rd.astype(np.float64).reshape(-1).tolist() == rows["rounded"]
    unb = O.linear_fp16_pipeline(*layer, round_output=False, bias=b)
    rdb = O.linear_fp16_pipeline(*layer, round_output=True, bias=b)
    assert unb.reshape(-1).tolist() == rows["unrounded_bias"]
    assert rdb.astype(np.float64).reshape(-1).tolist() == rows["rounded_bias"]
    # the exact layer does not round X': the ties above do not arise there
    assert np.allclose(O.linear(*layer).reshape(-1), rows["exact"], rtol=0, atol=1e-15)


# ---- the other group sizes (CSDN article, section 5.2: 64 and 256) ---------
@pytest.mark.parametrize("group", [64, 256])
def test_group_sizes_keep_the_structure(group):
    """At group 64 and 256: the rotation stays inside each group (a vector
    nonzero in one group only stays so), preserves each group's norm when
    alpha = 1, and (X T^-1)(T W) = X W; pairs reaching across a group are
    refused."""
    in_f = 512
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed=group, pairs_per_group=group // 2, group=group)
    x = synth.activations(6, in_f, seed=group).astype(np.float64)
    ones = np.ones(in_f, np.float32)
    xr = O.rotate_activations(x, pairs, theta, ones, group)
    G = in_f // group
    assert np.allclose(np.linalg.norm(x.reshape(6, G, group), axis=2), np.linalg.norm(xr.reshape(6, G, group), axis=2),
                       rtol=1e-13)
    one = np.zeros((1, in_f))
    one[0, group:2 * group] = x[0, group:2 * group]
    r1 = O.rotate_activations(one, pairs, theta, alpha, group)
    assert np.all(r1[0, :group] == 0) and np.all(r1[0, 2 * group:] == 0) and np.any(r1[0, group:2 * group] != 0)
    w = synth.weight(32, in_f, seed=group).astype(np.float64)
    lhs = O.rotate_activations(x, pairs, theta, alpha, group) @ O.transform_weight(w, pairs, theta, alpha, group).T
    assert np.linalg.norm(lhs - x @ w.T) / np.linalg.norm(x @ w.T) < 1e-12
    bad = pairs.copy()
    bad[0, 0, 0] = (0, group)                         # channel index outside its group
    with pytest.raises(AssertionError):
        O.rotate_activations(np.zeros((1, in_f)), bad, theta, alpha, group)


@pytest.mark.parametrize("group", [64, 256])
def test_group_sizes_pairwise_match_the_dense_matrix(group):
    """Pairwise application against the independently built dense
    block-diagonal T, at the real group sizes (two groups)."""
    in_f = 2 * group
    pairs, theta, alpha = synth.rotation_params(in_f, 4, seed=group + 1, pairs_per_group=group // 2, group=group)
    T = O.dense_transform(pairs, theta, alpha, group=group)
    assert np.all(T[:group, group:] == 0) and np.all(T[group:, :group] == 0)
    x = np.random.default_rng(group).standard_normal((3, in_f))
    assert np.allclose(O.rotate_activations(x, pairs, theta, alpha, group), x @ np.linalg.inv(T), atol=1e-11)


@pytest.mark.parametrize("group", [64, 256])
def test_rtn_invariants_other_group_sizes(group):
    w = synth.weight(16, 512, seed=group).astype(np.float64)
    q, s, z = O.rtn_quantize(w, group=group)
    assert s.shape == (16, 512 // group) and z.shape == s.shape
    sf = np.repeat(s.astype(np.float64), group, axis=1)
    zf = np.repeat(z.astype(np.float64), group, axis=1)
    exact = (q - zf) * sf
    unclipped = (q > 0) & (q < 15)
    assert np.all(np.abs(w - exact)[unclipped] <= sf[unclipped] / 2 * (1 + 1e-12))
    # w_hat is the fp16 value nearest the exact product: within half the
    # spacing above |w_hat| (the larger one where w_hat sits on a power of two)
    wh = O.dequantize(q, s, z, group=group).astype(np.float64)
    spacing = np.spacing(np.abs(wh).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(wh - exact) <= spacing / 2)
