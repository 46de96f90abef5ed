"""Tolerance checks shared by the GPU parity tests (the bars are stated in
test_gpu_parity.py's docstring). Figures are recorded for the end-of-run
summary printed by conftest."""
import os

import numpy as np

import synth
from oracle import paro_oracle as O

ROT_TOL = 1e-3
REL_TOL = 2e-3
ABS_TOL = 1e-2
ACC_BUDGET = 2e-3


def _record(what, value, bound):
    import conftest
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]
    conftest.PARITY.append((test, what, float(value), bound))


def check_rotation(got16, x, pairs, theta, alpha, group=128):
    ref = O.rotate_activations(x, pairs, theta, alpha, group)
    fl, lit = O.rotation_rel_error(got16.astype(np.float64), ref)
    _record("X' rel err (floored 1% group max)", fl, ROT_TOL)
    _record("X' rel err (literal, ref != 0)", lit, "reported")
    assert fl <= ROT_TOL, (fl, lit)
    return fl


def output_bound(y, ref, x16):
    """Per-element bar: max(1e-2, |Y_x16 - Y_ref| + spacing16/2 + 2e-3)."""
    mag = np.maximum(np.abs(y), np.abs(ref)).astype(np.float16)
    half = 0.5 * np.abs(np.spacing(mag)).astype(np.float64)
    return np.maximum(ABS_TOL, np.abs(x16 - ref) + half + ACC_BUDGET)


def check_linear(y16, x, pairs, theta, alpha, q, s, z, bias=None, group=128):
    if pairs is None:                       # unrotated layer: theta = 0, alpha = 1
        pairs, theta, alpha = synth.rotation_params(x.shape[1], 1, 0, group=group)
        theta = np.zeros_like(theta)
        alpha = np.ones_like(alpha)
    ref = O.linear(x, pairs, theta, alpha, q, s, z, group=group, bias=bias)
    x16 = O.linear_fp16_pipeline(x, pairs, theta, alpha, q, s, z, group=group, round_output=False, bias=bias)
    floor = O.linear_fp16_pipeline(x, pairs, theta, alpha, q, s, z, group=group, round_output=True, bias=bias)
    y = y16.astype(np.float64)
    rel, mx = O.output_errors(y, ref)
    bound = output_bound(y, ref, x16)
    excess = np.abs(y - ref) - bound
    worst = float(np.max(excess)) if y.size else 0.0
    fmt = float(np.max(np.abs(floor.astype(np.float64) - ref))) if y.size else 0.0
    _record("Y rel Frobenius err", rel, REL_TOL)
    _record("Y max |dY|", mx, ABS_TOL)
    _record("Y max |dY| of the ideal fp16 pipeline", fmt, "format floor")
    assert rel <= REL_TOL, (rel, mx)
    assert worst <= 0.0, (rel, mx, worst, fmt)
    return rel, mx
