"""The seeded synthetic workloads follow their stated recipe (CPU only).

These generators feed both the CUDA path and the oracle, so their shapes, seeds and distributions
are what every parity case and bench line is measured on.  Checked here: the layer shapes and
element counts of the Llama-2-7B- and 70B-shaped sets, seeding (same seed, same values; different
workloads, different values), the moments of each distribution on small samples, the outlier
columns of the activation workload, and the oracle's host view of a tensor.
"""
import math

import numpy as np
import pytest
import torch

from fp4_microscaling_tensor_b200 import inputs


def test_layer_shapes_and_sizes():
    # Llama-2-70B layer: q and o 8192x8192, k and v 1024x8192 (grouped-query attention), and the
    # three MLP matrices, all taken as 8192x28672 (the element count of gate, up and down)
    assert inputs.LLAMA70B_SHAPES == [(8192, 8192)] * 2 + [(1024, 8192)] * 2 + [(8192, 28672)] * 3
    assert sum(r * c for r, c in inputs.LLAMA70B_SHAPES) == 855_638_016
    # Llama-2-7B layer: four 4096x4096 attention projections, three 4096x11008 MLP matrices
    assert inputs.LLAMA7B_SHAPES == [(4096, 4096)] * 4 + [(4096, 11008)] * 3
    assert 32 * sum(r * c for r, c in inputs.LLAMA7B_SHAPES) == 6_476_005_376
    # every row splits into whole blocks of every swept size
    for r, c in inputs.LLAMA70B_SHAPES + inputs.LLAMA7B_SHAPES:
        assert all(c % n == 0 for n in inputs.SWEEP_BLOCKS)


def test_seeding():
    a = inputs.normal((64, 64), 0.02, 7)
    assert torch.equal(a, inputs.normal((64, 64), 0.02, 7))
    assert not torch.equal(a, inputs.normal((64, 64), 0.02, 8))
    # the sweep's five sigmas draw from five seeds, so they are not rescaled copies of one draw
    w0 = inputs.workload2(0, shape=(32, 64)).float() / inputs.SWEEP_SIGMAS[0]
    w1 = inputs.workload2(1, shape=(32, 64)).float() / inputs.SWEEP_SIGMAS[1]
    assert not torch.allclose(w0, w1, rtol=0.05)
    # layers and tensors of a layer get distinct seeds
    t00 = inputs.workload5_tensor(0, 0, shape=(16, 64))
    assert not torch.equal(t00, inputs.workload5_tensor(0, 1, shape=(16, 64)))
    assert not torch.equal(t00, inputs.workload5_tensor(1, 0, shape=(16, 64)))
    assert torch.equal(inputs.workload3_tensor(2, 3, shape=(16, 64)),
                       inputs.workload3_tensor(2, 3, shape=(16, 64)))


@pytest.mark.parametrize("sigma", inputs.SWEEP_SIGMAS)
def test_normal_moments(sigma):
    x = inputs.normal((512, 512), sigma, 11).double()
    assert abs(x.mean().item()) < 5 * sigma / 512
    assert abs(x.std().item() / sigma - 1.0) < 0.01


def test_workload1_is_fp32_and_workload5_is_bf16():
    w1 = inputs.workload1()
    assert w1.dtype == torch.float32 and w1.shape == (256, 256)
    assert abs(w1.std().item() / 0.02 - 1.0) < 0.02
    w5 = inputs.workload5_tensor(0, 0, shape=(256, 256))
    assert w5.dtype == torch.bfloat16
    assert abs(w5.float().std().item() / 0.015 - 1.0) < 0.02


def test_student_t_rowgain_moments():
    sigma = 0.02
    x = inputs.student_t4_rowgain((2048, 1024), 5, sigma=sigma).double()
    # t with 4 degrees of freedom has variance 2, rescaled to sigma^2; the row gain exp(0.5 Z) has
    # E[gain^2] = e^0.5
    ms = (x * x).mean().item()
    assert abs(ms / (sigma * sigma * math.exp(0.5)) - 1.0) < 0.25
    # heavy tails: t4 has infinite kurtosis, so the sample excess kurtosis of rows scaled to unit
    # variance (which removes the row gain) is far above a normal's 0
    rows = x / x.std(dim=1, keepdim=True)
    kurt = ((rows ** 4).mean(dim=1) - 3.0).mean().item()
    assert kurt > 1.0
    # per-row gains differ: row RMS spreads like a log-normal(0, 0.5) factor
    rms = torch.sqrt((x * x).mean(dim=1))
    spread = torch.log(rms).std().item()
    assert 0.35 < spread < 0.65


def test_activation_outlier_columns():
    x = inputs.activation_outliers(shape=(256, 8192)).float()
    col_std = x.std(dim=0)
    big = col_std > 10.0
    assert int(big.sum()) == round(0.01 * 8192) == 82
    assert abs(col_std[big].mean().item() / 50.0 - 1.0) < 0.1
    assert abs(col_std[~big].mean().item() - 1.0) < 0.05
    # the outlier columns do not depend on the row count (a separate seeded permutation)
    y = inputs.activation_outliers(shape=(64, 8192)).float()
    assert torch.equal(big, y.std(dim=0) > 10.0)


def test_to_oracle_views():
    x = inputs.normal((8, 16), 0.5, 3)
    v = inputs.to_oracle(x)
    assert v.dtype == np.uint16 and v.shape == (128,)
    assert np.array_equal(v, x.view(torch.int16).numpy().view(np.uint16).reshape(-1))
    f = inputs.workload1()
    assert np.array_equal(inputs.to_oracle(f), f.numpy().reshape(-1))
    with pytest.raises(TypeError):
        inputs.to_oracle(torch.zeros(4, dtype=torch.float16))
