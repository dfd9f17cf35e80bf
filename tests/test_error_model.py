"""The analytic three-term error model shipped with the library (`error_model.py`).

On the CPU it must equal, over a grid of sigma x N x format, the quadrature of
test_oracle_error_model.py -- computed by a different method (two-level Gauss-Legendre, no closed
forms) and itself pinned to the oracle by Monte Carlo -- and it is pinned directly by Monte Carlo
against the oracle's error reduction on Gaussian samples.  It must reproduce the pages'
narrow-tensor claim (the zero-scale term dominates small E4M3 blocks, UE5M3 removes it).  On the
GPU the measured terms of the fused pass on bf16 4096x4096 N(0, sigma^2) tensors must match the
model within the sampling error of 16.8 M values (2% of the total; 5% of a term that is at least
1% of the total).
"""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from fp4_microscaling_tensor_b200 import error_model as em  # noqa: E402

CASES = [(0.005, 4, em.E4M3), (0.005, 4, em.UE5M3), (0.02, 32, em.E4M3), (0.02, 32, em.UE5M3),
         (0.1, 256, em.E4M3), (0.01, 16, em.UE5M3)]


@pytest.mark.parametrize("sigma,N,fmt", CASES)
def test_model_equals_independent_quadrature(sigma, N, fmt):
    import test_oracle_error_model as ref
    a, b = em.model(sigma, N, fmt), ref.model(sigma, N, fmt)
    tot = sum(b.values())
    for k in ("elem", "max", "zero"):
        assert abs(a[k] - b[k]) <= 1e-9 * tot, (k, a[k], b[k])


@pytest.mark.parametrize("sigma,N,fmt", [(0.005, 4, em.E4M3), (0.02, 32, em.UE5M3),
                                         (0.1, 256, em.E4M3)])
def test_model_matches_oracle_monte_carlo(sigma, N, fmt):
    """The shipped model against the oracle's sums on 2M seeded Gaussian values (32 chunks)."""
    import test_oracle_error_model as ref
    mod = em.model(sigma, N, fmt)
    mc = ref.monte_carlo(sigma, N, fmt, seed=77)
    total = sum(mod.values())
    for k in ("elem", "max", "zero"):
        mean, se = mc[k]
        assert abs(mean - mod[k]) <= 4 * se + 1e-3 * abs(mod[k]) + 1e-9 * total, (k, mean, mod[k])


def test_narrow_tensor_claim():
    e4, ue = em.model(0.005, 4, em.E4M3), em.model(0.005, 4, em.UE5M3)
    assert e4["zero"] > e4["elem"] + e4["max"]
    assert ue["zero"] < 1e-6 * (ue["elem"] + ue["max"])


@pytest.mark.gpu
@pytest.mark.parametrize("sigma,N,fmt", CASES)
def test_measured_terms_match_model(cuda_device, sigma, N, fmt):
    import fp4_microscaling_tensor_b200 as mx
    from fp4_microscaling_tensor_b200 import inputs
    x = inputs.workload2(em.SIGMAS.index(sigma), device=cuda_device)
    st = mx.quantize_with_stats(x, N, fmt)[2].to_dict()
    got = {"elem": st["mse_elem"], "max": st["mse_max"], "zero": st["mse_zero"]}
    mod = em.model(sigma, N, fmt)
    tot = sum(mod.values())
    assert abs(sum(got.values()) - tot) <= 0.02 * tot, (got, mod)
    for k in ("elem", "max", "zero"):
        if mod[k] >= 0.01 * tot:
            assert abs(got[k] - mod[k]) <= 0.05 * mod[k], (k, got[k], mod[k])
        else:
            assert got[k] <= 0.02 * tot, (k, got[k], mod[k])


def test_adaptive_block_size_rule():
    assert [em.adaptive_block_size(s) for s in (0.001, 0.0099, 0.01, 0.05, 0.0999, 0.1, 1.0)] == \
        [128, 128, 64, 64, 64, 32, 32]


def test_model_block_size():
    # wide tensors: smaller blocks are more accurate; narrow E4M3 tensors: the zero-scale term
    # makes the smallest blocks worst (the pages' anomaly), UE5M3 removes it
    assert em.model_block_size(0.1, em.E4M3) == 4
    assert em.model_block_size(0.005, em.E4M3) > 4
    assert em.model_block_size(0.005, em.UE5M3) == 4
    # a storage budget of 4.25 bits per element allows N >= 32 only
    n = em.model_block_size(0.1, em.E4M3, max_bits=4.25)
    assert n == 32 and em.bits_per_element(n) <= 4.25
    with pytest.raises(ValueError):
        em.model_block_size(0.1, em.E4M3, max_bits=4.0)
