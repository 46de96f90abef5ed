"""CPU fp64 oracle for ParoQuant's rotated W4G128 linear layer.

TEST INFRASTRUCTURE ONLY. Only the test suite, the package entry's smoke
check and the benchmark's CPU-baseline leg may import this module. The CUDA
library never calls it and shares no code with it.

What is computed, and where the pages define it
-----------------------------------------------
ParoQuant paper notes (ICLR 2026 notes page), "key design":
  * a Givens rotation of a channel pair (i, j) updates the rows of W as
        W[i,:] <- cos(th) W[i,:] - sin(th) W[j,:]
    and (CSDN article, section 2.2, the 2x2 matrix) jointly
        [v_i']   [cos -sin] [v_i]
        [v_j'] = [sin  cos] [v_j];
  * "independent rotation": every channel is in at most one pair of a layer,
    and pairs stay inside one quantisation group;
  * K layers (K = 8 by default) and a channel scaling form the transform
        T = (prod_{t=1..K} R(P_t, Theta_t)) * diag(alpha).
CSDN article, section 2.1: Y = X W + b = (X T^-1)(T W) + b.

Orientation: the pages write Y = X W with W of shape [in][out]; T acts on the
input channels (rows of that W). Here weights are stored [out][in] (PyTorch
orientation), so T acts along the last axis of every output row.

Readings where the pages leave a step open:
  * product order: layer t = 1 is applied first after diag(alpha), i.e.
    T = R_K ... R_1 diag(alpha) (the CSDN pseudo-code scales first, then
    rotates in list order);
  * activations: X T^-1 = X diag(1/alpha) R_1^T ... R_K^T, which per row is
    "divide by alpha, then layers t = 1..K with the same 2x2 formula";
  * quantiser: asymmetric round-to-nearest-even per 128-input group,
    s = fp16((max - min) / 15) floored at 2^-14, z = clamp(rint(-min/s), 0, 15),
    q = clamp(rint(w/s) + z, 0, 15), using the stored fp16 s;
  * dequantised weight: w_hat = fp16((q - z) * s) (the exact product rounded
    once to fp16).
"""
from __future__ import annotations

import numpy as np

GROUP = 128
S_FLOOR = 2.0 ** -14          # smallest normal fp16; floor for degenerate groups


# --------------------------------------------------------------------------
# Rotation layers
# --------------------------------------------------------------------------
def _check_pairs(pairs: np.ndarray, in_features: int, group: int) -> None:
    """Independence and group locality (paper notes, "independent rotation")."""
    K, G, P, two = pairs.shape
    assert two == 2 and G * group == in_features, "pairs must be [K][in/group][P][2]"
    for t in range(K):
        for g in range(G):
            idx = pairs[t, g].reshape(-1).astype(np.int64)
            assert idx.min() >= 0 and idx.max() < group, "pair index outside its group"
            assert len(np.unique(idx)) == idx.size, "a channel appears in two pairs of one layer"


def givens_layer(v: np.ndarray, pairs_t: np.ndarray, theta_t: np.ndarray, group: int = GROUP) -> np.ndarray:
    """Apply one independent rotation layer R(P_t, Theta_t) along the last axis.

    pairs_t: [G][P][2] group-local indices; theta_t: [G][P].
    Every pair (i, j) with angle th maps (v_i, v_j) to
    (cos th v_i - sin th v_j, sin th v_i + cos th v_j); pairs are disjoint, so
    all of them read the layer's input (CSDN article, section 2.2).
    """
    out = np.array(v, dtype=np.float64, copy=True)
    G, P, _ = pairs_t.shape
    base = (np.arange(G) * group)[:, None]
    i = (base + pairs_t[:, :, 0].astype(np.int64)).reshape(-1)
    j = (base + pairs_t[:, :, 1].astype(np.int64)).reshape(-1)
    th = theta_t.astype(np.float64).reshape(-1)      # cos/sin in fp64 of the fp32 angle
    c, s = np.cos(th), np.sin(th)
    vi, vj = v[..., i].astype(np.float64), v[..., j].astype(np.float64)
    out[..., i] = c * vi - s * vj
    out[..., j] = s * vi + c * vj
    return out


def transform_weight(w: np.ndarray, pairs: np.ndarray, theta: np.ndarray, alpha: np.ndarray,
                     group: int = GROUP) -> np.ndarray:
    """W' = T W along the input axis: scale channel c by alpha_c, then layers t = 1..K."""
    w = np.asarray(w, dtype=np.float64)
    _check_pairs(pairs, w.shape[-1], group)
    v = w * alpha.astype(np.float64)
    for t in range(pairs.shape[0]):
        v = givens_layer(v, pairs[t], theta[t], group)
    return v


def rotate_activations(x: np.ndarray, pairs: np.ndarray, theta: np.ndarray, alpha: np.ndarray,
                       group: int = GROUP) -> np.ndarray:
    """X' = X T^-1 = X diag(1/alpha) R_1^T ... R_K^T, row by row.

    x R^T is (R x^T)^T, so each layer uses the same 2x2 formula as the weight
    side, in the same order t = 1..K, after dividing channel c by alpha_c.
    """
    x = np.asarray(x, dtype=np.float64)
    _check_pairs(pairs, x.shape[-1], group)
    v = x / alpha.astype(np.float64)
    for t in range(pairs.shape[0]):
        v = givens_layer(v, pairs[t], theta[t], group)
    return v


def dense_transform(pairs: np.ndarray, theta: np.ndarray, alpha: np.ndarray, group: int = GROUP) -> np.ndarray:
    """The dense [in][in] matrix T = R_K ... R_1 diag(alpha), built as a product
    of explicit Givens matrices (identity with (i,i)=c, (i,j)=-s, (j,i)=s,
    (j,j)=c per pair). Used by tests on small sizes only."""
    K, G, P, _ = pairs.shape
    n = G * group
    T = np.diag(alpha.astype(np.float64))
    for t in range(K):
        R = np.eye(n)
        for g in range(G):
            for p in range(P):
                i = g * group + int(pairs[t, g, p, 0])
                j = g * group + int(pairs[t, g, p, 1])
                th = float(np.float64(theta[t, g, p]))
                c, s = np.cos(th), np.sin(th)
                R[i, i], R[i, j], R[j, i], R[j, j] = c, -s, s, c
        T = R @ T
    return T


# --------------------------------------------------------------------------
# W4G128 asymmetric round-to-nearest quantiser and dequantiser
# --------------------------------------------------------------------------
def rtn_quantize(w: np.ndarray, group: int = GROUP):
    """Per (row, 128-input group): q uint8 [out][in], s fp16 [out][G], z uint8 [out][G].

    s = fp16((max - min) / 15), replaced by 2^-14 when it is below the smallest
    normal fp16 (degenerate groups); z = clamp(rint(-min / s), 0, 15);
    q = clamp(rint(w / s) + z, 0, 15). Rounding is half-to-even; s is the
    stored fp16 value.
    """
    w = np.asarray(w, dtype=np.float64)
    out, n = w.shape
    assert n % group == 0
    G = n // group
    wg = w.reshape(out, G, group)
    mn, mx = wg.min(axis=2), wg.max(axis=2)
    s16 = ((mx - mn) / 15.0).astype(np.float16)
    if not np.all(np.isfinite(s16)):
        raise OverflowError("group range does not fit an fp16 scale")
    s = s16.astype(np.float64)
    s = np.where(s < S_FLOOR, S_FLOOR, s)
    s16 = s.astype(np.float16)
    z = np.clip(np.rint(-mn / s), 0, 15)
    q = np.clip(np.rint(wg / s[:, :, None]) + z[:, :, None], 0, 15)
    return q.reshape(out, n).astype(np.uint8), s16, z.astype(np.uint8)


def dequantize(q: np.ndarray, s: np.ndarray, z: np.ndarray, group: int = GROUP) -> np.ndarray:
    """w_hat fp16 [out][in] = fp16((q - z) * s): exact product, one rounding."""
    out, n = q.shape
    G = n // group
    d = q.reshape(out, G, group).astype(np.float64) - z.astype(np.float64)[:, :, None]
    prod = d * s.astype(np.float64)[:, :, None]
    return prod.reshape(out, n).astype(np.float16)


def quantize_layer(w: np.ndarray, pairs, theta, alpha, group: int = GROUP):
    """Offline step: W' = T W, then RTN. Returns (q, s, z, W')."""
    wt = transform_weight(w, pairs, theta, alpha, group)
    q, s, z = rtn_quantize(wt, group)
    return q, s, z, wt


# --------------------------------------------------------------------------
# The layer
# --------------------------------------------------------------------------
def linear(x: np.ndarray, pairs, theta, alpha, q, s, z, group: int = GROUP, bias=None) -> np.ndarray:
    """Y = (X T^-1) w_hat^T (+ b) in fp64, unrounded. x fp16/fp64 [T][in] -> [T][out].
    The bias b [out] is the "+ b" of CSDN article section 2.1 (Y = XW + b)."""
    xr = rotate_activations(x, pairs, theta, alpha, group)
    y = xr @ dequantize(q, s, z, group).astype(np.float64).T
    return y if bias is None else y + np.asarray(bias, dtype=np.float64)[None, :]


def linear_fp16_pipeline(x: np.ndarray, pairs, theta, alpha, q, s, z, group: int = GROUP,
                         round_output: bool = True, bias=None) -> np.ndarray:
    """The ideal fp16 pipeline: X' rounded to fp16, fp64 contraction with w_hat
    (+ b), Y rounded to fp16 (or left in fp64 with round_output=False). Its
    distance to `linear` is the format floor of any kernel that stores X' and
    Y in fp16."""
    xr = rotate_activations(x, pairs, theta, alpha, group).astype(np.float16).astype(np.float64)
    y = xr @ dequantize(q, s, z, group).astype(np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y.astype(np.float16) if round_output else y


# --------------------------------------------------------------------------
# Error measures used by the parity tests
# --------------------------------------------------------------------------
def rotation_rel_error(got: np.ndarray, ref: np.ndarray, group: int = GROUP, floor: float = 1e-2):
    """Per-element |got - ref| / max(|ref|, floor * max_{c in group} |ref_c|).

    Returns (max floored relative error, max literal relative error over
    elements with ref != 0)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    T, n = ref.shape
    gmax = np.abs(ref).reshape(T, n // group, group).max(axis=2)
    den = np.maximum(np.abs(ref), floor * np.repeat(gmax, group, axis=1))
    err = np.abs(got - ref)
    floored = float(np.max(err / np.where(den > 0, den, 1.0))) if ref.size else 0.0
    nz = ref != 0
    literal = float(np.max(err[nz] / np.abs(ref[nz]))) if np.any(nz) else 0.0
    return floored, literal


def output_errors(got: np.ndarray, ref: np.ndarray):
    """(||got - ref||_F / ||ref||_F, max |got - ref|)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0, 0.0
    nrm = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (nrm if nrm > 0 else 1.0)), float(np.max(np.abs(got - ref)))
