"""Seeded synthetic inputs for the rotated W4G128 linear layer.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no rotation, no transform, no quantisation). Both the
CPU oracle (tests) and the CUDA path (tests, bench) take their inputs from
here, so the two sides see identical bytes.

Distributions follow the workloads described for ParoQuant's evaluation
(Llama-3-8B / Qwen3 shaped layers, "ParoQuant: Pairwise Rotation
Quantization ..." paper notes, main-experiment table):

* activations X  ~ N(0, 1) fp16, with 4 seeded outlier channels scaled x20;
* weights W      ~ N(0, 0.02) fp16, with 1% of the input channels scaled x20;
* per rotation layer t and 128-channel group g, a uniform random perfect
  matching of the group's channels (Fisher-Yates permutation, paired as
  (perm[2p], perm[2p+1])); the partial variant keeps the first P pairs;
* angles theta ~ U(-pi, pi) (fp32), channel scales alpha = exp(N(0, 0.3))
  (fp32).

Every generator takes an integer seed and a stream id, combined through
numpy's PCG64 SeedSequence; the same (seed, stream) always yields the same
array on any machine.
"""
from __future__ import annotations

import numpy as np

GROUP = 128

# stream ids: independent random streams per input kind
_S_X, _S_X_OUT, _S_W, _S_W_OUT, _S_PAIRS, _S_THETA, _S_ALPHA = range(7)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


def activations(tokens: int, in_features: int, seed: int,
                n_outliers: int = 4, outlier_scale: float = 20.0) -> np.ndarray:
    """X fp16 [tokens][in_features]: N(0,1) with `n_outliers` channels x`outlier_scale`."""
    x = _rng(seed, _S_X).standard_normal((tokens, in_features))
    if n_outliers > 0 and in_features > 0:
        ch = _rng(seed, _S_X_OUT).choice(in_features, size=min(n_outliers, in_features), replace=False)
        x[:, ch] *= outlier_scale
    return x.astype(np.float16)


def weight(out_features: int, in_features: int, seed: int,
           outlier_frac: float = 0.01, outlier_scale: float = 20.0, std: float = 0.02) -> np.ndarray:
    """W fp16 [out_features][in_features] (PyTorch orientation): N(0, std) with
    `outlier_frac` of the input channels scaled x`outlier_scale`."""
    w = _rng(seed, _S_W).standard_normal((out_features, in_features)) * std
    n_out = int(round(outlier_frac * in_features))
    if n_out > 0:
        ch = _rng(seed, _S_W_OUT).choice(in_features, size=n_out, replace=False)
        w[:, ch] *= outlier_scale
    return w.astype(np.float16)


def matchings(in_features: int, K: int, seed: int, pairs_per_group: int = GROUP // 2,
              group: int = GROUP) -> np.ndarray:
    """Pair tables int16 [K][G][P][2] of group-local channel indices.

    For every (t, g) a uniform random permutation of 0..group-1 is drawn and
    paired as (perm[2p], perm[2p+1]); the first `pairs_per_group` pairs are
    kept (all group/2 for a perfect matching, fewer for the partial variant).
    """
    if in_features % group:
        raise ValueError("in_features must be a multiple of the group size")
    G = in_features // group
    if not 0 < pairs_per_group <= group // 2:
        raise ValueError("pairs_per_group out of range")
    rng = _rng(seed, _S_PAIRS)
    out = np.empty((K, G, pairs_per_group, 2), dtype=np.int16)
    for t in range(K):
        for g in range(G):
            perm = rng.permutation(group)              # numpy's Fisher-Yates shuffle
            out[t, g] = perm[: 2 * pairs_per_group].reshape(pairs_per_group, 2)
    return out


def angles(K: int, G: int, pairs_per_group: int, seed: int) -> np.ndarray:
    """theta fp32 [K][G][P] ~ U(-pi, pi)."""
    return _rng(seed, _S_THETA).uniform(-np.pi, np.pi, (K, G, pairs_per_group)).astype(np.float32)


def channel_scales(in_features: int, seed: int, sigma: float = 0.3) -> np.ndarray:
    """alpha fp32 [in_features] = exp(N(0, sigma))."""
    return np.exp(_rng(seed, _S_ALPHA).normal(0.0, sigma, in_features)).astype(np.float32)


def rotation_params(in_features: int, K: int, seed: int, pairs_per_group: int = GROUP // 2,
                    group: int = GROUP):
    """(pairs, theta, alpha) for one layer, all from `seed`."""
    G = in_features // group
    return (matchings(in_features, K, seed, pairs_per_group, group),
            angles(K, G, pairs_per_group, seed),
            channel_scales(in_features, seed))


_S_CODES = 7


def w4_codes(out_features: int, in_features: int, seed: int, group: int = GROUP):
    """Random valid W4G128 codes, not derived from any weight: q uint8 [out][in]
    ~ U{0..15}, z uint8 [out][in/group] ~ U{0..15}, s fp16 [out][in/group]
    ~ U(0.002, 0.02). Used where a test needs the layer's inputs at full size
    without running the offline quantiser."""
    rng = _rng(seed, _S_CODES)
    G = in_features // group
    q = rng.integers(0, 16, (out_features, in_features), dtype=np.uint8)
    z = rng.integers(0, 16, (out_features, G), dtype=np.uint8)
    s = rng.uniform(0.002, 0.02, (out_features, G)).astype(np.float16)
    return q, s, z


def layer_seed(config_id: int, layer_id: int) -> int:
    """Seed convention: 1000 * config id + layer id."""
    return 1000 * int(config_id) + int(layer_id)
