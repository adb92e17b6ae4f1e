"""Helpers shared by the GPU parity tests: seeded device inputs, the oracle on
the same bytes, and the tolerances.

Tolerances: fp32 inputs -> max |diff| <= 1e-4; bf16 inputs with fp32
accumulation -> max |diff| <= 1e-2 and mean |diff| <= 1e-3, compared on fp32
outputs (bf16 rounding of the output itself is checked separately).
"""
import math

import numpy as np

from long_context_attention_pair_b200 import synthetic

TOL_F32_MAX = 1e-4
TOL_BF16_MAX = 1e-2
TOL_BF16_MEAN = 1e-3


def gen(seed, name, shape, dtype, device="cuda"):
    return synthetic.tensor_torch(seed, name, shape, dtype, device=device)


def host(t):
    return t.float().cpu().numpy()


def check(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx, mean = float(err.max()), float(err.mean())
    if dtype == "f32":
        assert mx <= TOL_F32_MAX, f"{what}: max |diff| {mx:.3e} > {TOL_F32_MAX}"
    else:
        assert mx <= TOL_BF16_MAX, f"{what}: max |diff| {mx:.3e} > {TOL_BF16_MAX}"
        assert mean <= TOL_BF16_MEAN, f"{what}: mean |diff| {mean:.3e} > {TOL_BF16_MEAN}"
    return mx, mean


def sample_rows(N, count, seed):
    """`count` distinct query rows, always including 0 and N-1."""
    rng = np.random.default_rng(seed)
    if N <= count:
        return np.arange(N)
    pick = rng.choice(np.arange(1, N - 1), size=count - 2, replace=False)
    return np.sort(np.concatenate([[0, N - 1], pick]))


INF = math.inf
