"""The fp32 accumulation of tcgen05.mma chains against exact sums, and the allowance the
certified k-means assignment takes for it.

The tensor-core assignment certifies a nearest centroid when the gap to the runner-up
exceeds a bound on the error of its scores; the bound allows ALLOWANCE units of 2^-23 per
16-channel MMA step, relative to the largest magnitude that step can hold (the running sum
of |products| up to the step's end bounds both the accumulator and the step's products).
That allowance is the worst case of the accumulation model of Fasi, Higham, Mikaitis and
Pranesh, "Numerical behavior of NVIDIA tensor cores" (PeerJ Comput. Sci. 7:e330, 2021):
exact products, aligned to the largest term and truncated, so each of a step's 16 products
and the accumulator loses less than one unit of the largest term (17), plus one unit for
the normalisation of the result (18).  NVIDIA documents no model for tcgen05, so this test
measures the hardware: chains of 16 and 32 steps (the k-means assignment at d = 128 runs
2 x 8 steps) on random, wide-exponent, cancelling and swamping operands, against sums that
are exact up to one binary64 rounding (math.fsum of products that are exact in binary64).
The measured worst case must stay below the allowance with a margin of 1.25.
"""
import math

import numpy as np
import pytest
import torch

from free_sparse_attention_b200 import capi

pytestmark = pytest.mark.gpu

ALLOWANCE = 18.0   # units of 2^-23 per step, as in bound_E of kmeans_tc.cu
MARGIN = 1.25


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from free_sparse_attention_b200.build import build
    build()
    capi.lib()


def _bf16(x):
    """float64 -> the nearest bf16 values (as a device bf16 tensor and exact float64)."""
    t = torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.cuda(), t.to(torch.float64).numpy()


def _operands(kind, K, N, rng):
    if kind == "normal":
        a, b = rng.standard_normal((128, K)), rng.standard_normal((N, K))
    elif kind == "wide_exponent":
        a = rng.choice([-1.0, 1.0], (128, K)) * np.exp2(rng.integers(-24, 25, (128, K))) * rng.uniform(1, 2, (128, K))
        b = rng.choice([-1.0, 1.0], (N, K)) * np.exp2(rng.integers(-24, 25, (N, K))) * rng.uniform(1, 2, (N, K))
    elif kind == "cancelling":
        # products in pairs +X, -X(1 - 2^-8 r): large magnitudes, small running sums
        a = rng.uniform(1, 2, (128, K)) * np.exp2(rng.integers(0, 12, (128, K)))
        b = np.empty((N, K))
        b[:, 0::2] = rng.uniform(1, 2, (N, K // 2))
        b[:, 1::2] = -b[:, 0::2] * (1 - np.exp2(-8) * rng.uniform(0, 1, (N, K // 2)))
        a[:, 1::2] = a[:, 0::2]
    elif kind == "swamping":
        # one huge product first, then many small same-sign products below its last bit
        a = rng.uniform(1, 2, (128, K)) * np.exp2(-10)
        b = rng.uniform(1, 2, (N, K))
        a[:, 0] = np.exp2(16)
        b[:, 0] = 1.0
    elif kind == "swamping_negative":
        a = rng.uniform(1, 2, (128, K)) * np.exp2(-10)
        b = -rng.uniform(1, 2, (N, K))
        a[:, 0] = np.exp2(16)
        b[:, 0] = 1.0
    else:
        raise ValueError(kind)
    return a, b


def _units(D, a, b):
    """Error of each output in units of 2^-23 per step of the running |product| sums."""
    K = a.shape[1]
    steps = K // 16
    out = np.empty(D.shape)
    for i in range(a.shape[0]):
        prod = a[i][None, :] * b                      # exact in binary64 (bf16 x bf16)
        absrun = np.cumsum(np.abs(prod), axis=1)      # exact enough: only scales the metric
        S = absrun[:, 15::16].sum(axis=1)             # sum over steps of the running magnitude
        exact = np.array([math.fsum(row) for row in prod])
        out[i] = np.abs(D[i] - exact) / (np.exp2(-23) * S)
    assert steps == K // 16
    return out


@pytest.mark.parametrize("K", [256, 512], ids=["16-steps", "32-steps"])
@pytest.mark.parametrize("kind", ["normal", "wide_exponent", "cancelling", "swamping", "swamping_negative"])
def test_accumulation_error_within_the_kmeans_allowance(kind, K):
    rng = np.random.default_rng(hash((kind, K)) % 2 ** 32)
    N = 64
    a, b = _operands(kind, K, N, rng)
    A, a = _bf16(a)
    B, b = _bf16(b)
    D = capi.tc_accumulation_probe(A, B).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    u = _units(D, a, b)
    worst = float(u.max())
    print(f"{kind} K={K}: worst {worst:.3f} units of 2^-23 per step (allowance {ALLOWANCE})")
    assert np.isfinite(D).all()
    assert worst * MARGIN <= ALLOWANCE, (kind, K, worst)
