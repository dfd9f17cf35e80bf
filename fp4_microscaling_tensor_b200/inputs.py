"""Seeded synthetic workloads (no method arithmetic here).

Both the CUDA path and the CPU oracle are fed from these generators: a tensor is drawn once (on the
device for the large workloads) and the oracle receives a host copy of the same values.  Shapes and
value distributions follow the five workloads the library is measured on:

1. fp32 256x256, N(0, 0.02^2), seed 0.
2. bf16 4096x4096, N(0, sigma^2) for sigma in SWEEP_SIGMAS, seed 100 + k (k = sigma index).
3. Llama-2-7B-shaped weight set: 32 layers x (4 of 4096x4096 + 3 of 4096x11008) bf16; Student-t
   with 4 degrees of freedom built from five normals as Z0 / sqrt((Z1^2+Z2^2+Z3^2+Z4^2)/4), rescaled
   by 0.02/sqrt(2) (its variance is 2) and multiplied by a per-row log-normal(0, 0.5) gain;
   seed 1000 + 7*layer + j.
4. activation-like bf16 16384x8192, N(0, 1) with 82 (1%) columns chosen by a seeded permutation
   multiplied by 50; seeds 2000 (values) and 2001 (columns).
5. Llama-2-70B-shaped layers: 2 of 8192x8192, 2 of 1024x8192, 3 of 8192x28672 bf16, N(0, 0.015^2);
   seed 3000 + 7*layer + j.
"""
import math

import torch

SWEEP_SIGMAS = (0.005, 0.01, 0.02, 0.05, 0.1)
SWEEP_BLOCKS = (4, 8, 16, 32, 64, 128, 256)
LLAMA7B_SHAPES = [(4096, 4096)] * 4 + [(4096, 11008)] * 3
LLAMA70B_SHAPES = [(8192, 8192)] * 2 + [(1024, 8192)] * 2 + [(8192, 28672)] * 3


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, sigma, seed, device="cpu", dtype=torch.bfloat16):
    """N(0, sigma^2) drawn in fp32 with the given seed, then rounded to dtype."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (x * sigma).to(dtype)


def student_t4_rowgain(shape, seed, sigma=0.02, device="cpu", dtype=torch.bfloat16):
    """Student-t (nu=4) with standard deviation sigma, times a per-row log-normal(0, 0.5) gain."""
    g = _gen(seed, device)
    rows, cols = shape
    z = [torch.randn(shape, generator=g, device=device, dtype=torch.float32) for _ in range(5)]
    t = z[0] / torch.sqrt((z[1] ** 2 + z[2] ** 2 + z[3] ** 2 + z[4] ** 2) / 4.0)
    gain = torch.exp(0.5 * torch.randn((rows, 1), generator=g, device=device, dtype=torch.float32))
    return (t * (sigma / math.sqrt(2.0)) * gain).to(dtype)


def activation_outliers(shape=(16384, 8192), seed=2000, chan_seed=2001, frac=0.01, gain=50.0,
                        device="cpu", dtype=torch.bfloat16):
    """N(0,1) activations with round(frac * hidden) seeded columns multiplied by `gain`."""
    rows, cols = shape
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    gc = _gen(chan_seed, "cpu")
    k = int(round(frac * cols))
    chans = torch.randperm(cols, generator=gc)[:k].to(device)
    x[:, chans] *= gain
    return x.to(dtype)


def workload1(device="cpu"):
    return normal((256, 256), 0.02, 0, device=device, dtype=torch.float32)


def workload2(sigma_index, shape=(4096, 4096), device="cpu"):
    return normal(shape, SWEEP_SIGMAS[sigma_index], 100 + sigma_index, device=device)


def workload3_tensor(layer, j, device="cpu", shape=None):
    shape = shape or LLAMA7B_SHAPES[j]
    return student_t4_rowgain(shape, 1000 + 7 * layer + j, device=device)


def workload4(device="cpu", shape=(16384, 8192)):
    return activation_outliers(shape, device=device)


def workload5_tensor(layer, j, device="cpu", shape=None):
    shape = shape or LLAMA70B_SHAPES[j]
    return normal(shape, 0.015, 3000 + 7 * layer + j, device=device)


def to_oracle(x):
    """Host numpy view for the oracle: uint16 bit patterns for bf16, float32 otherwise."""
    x = x.detach().contiguous().cpu()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view("uint16").reshape(-1)
    if x.dtype == torch.float32:
        return x.numpy().reshape(-1)
    raise TypeError(f"unsupported dtype {x.dtype}")
