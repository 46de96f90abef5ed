"""The output bar of the GPU parity tests, checked on the CPU with simulated
kernel outputs: a correctly rounded fp16 result of an fp32 sum passes; one
rounded to the wrong fp16 neighbour fails unless the exact value lies within
the 2e-3 budget (plus the X' rounding effect, twice) of a rounding midpoint;
an error of 1e-2 on a small output fails."""
import numpy as np

import synth
from oracle import paro_oracle as O
from parity import output_bound


def _layer(T=6, in_f=512, out_f=64, seed=3, x_scale=8.0):
    pairs, theta, alpha = synth.rotation_params(in_f, 8, seed)
    q, s, z = synth.w4_codes(out_f, in_f, seed)
    s = (s.astype(np.float32) * 40).astype(np.float16)          # outputs up to a few hundred
    x = (synth.activations(T, in_f, seed).astype(np.float32) * x_scale).astype(np.float16)
    ref = O.linear(x, pairs, theta, alpha, q, s, z)
    x16 = O.linear_fp16_pipeline(x, pairs, theta, alpha, q, s, z, round_output=False)
    return ref, x16


def test_correct_rounding_passes():
    ref, x16 = _layer()
    assert np.abs(ref).max() > 64                                # spacing >= 2^-4 somewhere
    noise = np.random.default_rng(0).uniform(-1e-3, 1e-3, ref.shape)   # fp32 accumulation
    y = (x16 + noise).astype(np.float16).astype(np.float64)
    assert np.all(np.abs(y - ref) <= output_bound(y, ref, x16))


def test_wrong_neighbour_fails():
    ref, x16 = _layer()
    y0 = x16.astype(np.float16)
    big = np.abs(y0.astype(np.float64)) >= 8.0                   # spacing >= 2^-7 ~ 7.8e-3
    assert big.sum() > 10
    # the other fp16 neighbour of the exact value: one step away from it
    away = np.where(y0.astype(np.float64) >= x16, -np.inf, np.inf).astype(np.float16)
    wrong = np.nextafter(y0, away).astype(np.float64)
    y = np.where(big, wrong, y0.astype(np.float64))
    ok = np.abs(y - ref) <= output_bound(y, ref, x16)
    half = 0.5 * np.abs(np.spacing(y0)).astype(np.float64)
    margin = half - np.abs(y0.astype(np.float64) - x16)          # distance of the value to the midpoint
    clear = big & (margin > 2 * np.abs(x16 - ref) + 2e-3 + 1e-9)
    assert clear.sum() > 20
    assert not np.any(ok[clear])


def test_small_output_keeps_the_absolute_bar():
    ref, x16 = _layer(x_scale=0.05)
    small = np.abs(ref) < 1.0
    assert small.sum() > 10
    y = ref + 1.05e-2
    ok = np.abs(y - ref) <= output_bound(y, ref, x16)
    assert not np.any(ok[small])
