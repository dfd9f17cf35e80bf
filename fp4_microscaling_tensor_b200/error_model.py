"""Analytic three-term error model of block FP4 microscaling for iid Gaussian inputs.

The microscaling article (hotelren.com/news/2192771, §2.2, Eqs. (1)-(3)) splits the mean squared
quantization error of N(0, sigma^2) data into three terms: the non-max elements of blocks with a
non-zero scale (MSE_elem, weight (N-1)/N), the max element of such blocks (MSE_max, weight 1/N: the
error left by rounding the scale) and the blocks whose scale rounds to zero (MSE_zero).  Every term
is an expectation over the block maximum M, whose CDF is (2 Phi(m/sigma) - 1)^N; given M = m the
scale is S(m) = RNE_fmt(m / (6 g)) * g, the max element's error is (m - S q(m/S))^2 with q the
nearest E2M1 magnitude, and the other N - 1 values are iid normals truncated to |x| < m.  The inner
expectations are closed forms in Phi and phi; the outer integral is adaptive quadrature split at
every scale and element rounding breakpoint.  The values are mean squared errors per element, the
quantities `sse_* / numel` of the library's error record estimate.

`python -m fp4_microscaling_tensor_b200.error_model` prints the model over the sweep grid
(sigma x N x format); with `--measure` it also runs the sweep on the GPU (bf16 4096x4096 tensors,
the fused quantize + error-reduction pass) and prints the measured terms beside the model.
"""
import argparse
import math
import sys

import numpy as np
from scipy import integrate
from scipy.special import ndtr

E4M3, UE5M3 = 0, 1
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MID = (E2M1[:-1] + E2M1[1:]) / 2
SIGMAS = (0.005, 0.01, 0.02, 0.05, 0.1)
BLOCKS = (4, 8, 16, 32, 64, 128, 256)


def scale_values(fmt):
    """Every finite non-negative value of the scale format, ascending (E4M3FN without NaN: bias 7,
    subnormals m 2^-9; UE5M3: 8-bit unsigned, bias 15, subnormals m 2^-17, no inf/NaN)."""
    vals = []
    if fmt == E4M3:
        for c in range(0x7F):
            e, m = c >> 3, c & 7
            vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    else:
        for c in range(0x100):
            e, m = c >> 3, c & 7
            vals.append(m * 2.0 ** -17 if e == 0 else (1 + m / 8) * 2.0 ** (e - 15))
    return np.array(vals)


def _phi(z):
    return np.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)


def _seg_sq_err(p, r, c, sigma):
    """int_p^r (x - c)^2 phi(x/sigma)/sigma dx."""
    a, b = p / sigma, r / sigma
    z2 = (ndtr(b) - b * _phi(b)) - (ndtr(a) - a * _phi(a))
    z1 = _phi(a) - _phi(b)
    z0 = ndtr(b) - ndtr(a)
    return sigma * sigma * z2 - 2 * sigma * c * z1 + c * c * z0


def _inner(m, S, sigma):
    """int_0^m (x - S q(x/S))^2 phi(x/sigma)/sigma dx, q = nearest E2M1 magnitude (saturating)."""
    edges = np.concatenate([[0.0], S * E2M1_MID, [np.inf]])
    tot = 0.0
    for k in range(8):
        lo, hi = edges[k], min(edges[k + 1], m)
        if hi <= lo:
            break
        tot += _seg_sq_err(lo, hi, S * E2M1[k], sigma)
    return tot


def _max_err(m, S):
    v = m / S
    k = min(int(np.searchsorted(E2M1_MID, v, side="left")), 7)
    return (m - S * E2M1[k]) ** 2


def model(sigma, N, fmt, g=1.0):
    """{'elem', 'max', 'zero'}: the three mean squared errors per element for N(0, sigma^2)."""
    V = scale_values(fmt) * g
    mids = (V[:-1] + V[1:]) / 2
    mhi = 9.0 * sigma
    # pieces of constant scale: S = V[k] while m / 6 lies between two scale midpoints; saturated
    # above the top one
    bps = [0.0] + [6 * t for t in mids if 6 * t < mhi] + [mhi]
    out = {"elem": 0.0, "max": 0.0, "zero": 0.0}
    eps = 1e-12 * sigma ** 2

    def dens(m, power):
        z = m / sigma
        return (2 * ndtr(z) - 1) ** power * 2 * _phi(z) / sigma

    for lo, hi in zip(bps[:-1], bps[1:]):
        S = V[min(int(np.searchsorted(mids, (lo + hi) / 12)), len(V) - 1)]
        if S == 0:
            def fz(m):
                z = m / sigma
                return dens(m, N - 1) * m * m + (N - 1) * dens(m, N - 2) * 2 * sigma ** 2 * (
                    ndtr(z) - z * _phi(z) - 0.5)
            out["zero"] += integrate.quad(fz, lo, hi, epsabs=eps, epsrel=1e-10, limit=200)[0]
            continue
        pts = [S * t for t in E2M1_MID if lo < S * t < hi] or None
        out["max"] += integrate.quad(lambda m: dens(m, N - 1) * _max_err(m, S), lo, hi,
                                     points=pts, epsabs=eps, epsrel=1e-10, limit=200)[0]
        out["elem"] += integrate.quad(lambda m: (N - 1) * dens(m, N - 2) * 2 * _inner(m, S, sigma),
                                      lo, hi, points=pts, epsabs=eps, epsrel=1e-10, limit=200)[0]
    # dens(m, N - 1) is the density of the block maximum divided by N, so each term above is
    # already a mean per element (the max element is 1 of N, the others N - 1 of N)
    return out


def adaptive_block_size(sigma):
    """The pages' dynamic block-size rule (microscaling article §6 item 2): 128 below sigma =
    0.01, 64 below 0.1, else 32."""
    if sigma < 0.01:
        return 128
    if sigma < 0.1:
        return 64
    return 32


def bits_per_element(N):
    """Storage per element: a 4-bit code plus an 8-bit scale per block of N."""
    return 4.0 + 8.0 / N


def model_block_size(sigma, fmt, g=1.0, max_bits=None, blocks=BLOCKS):
    """The block size with the smallest modelled total MSE for N(0, sigma^2) data, among those
    whose storage (4 + 8/N bits per element) is at most max_bits (all when None); ties go to the
    larger block (less storage)."""
    best = None
    for n in sorted(blocks, reverse=True):
        if max_bits is not None and bits_per_element(n) > max_bits:
            continue
        tot = sum(model(sigma, n, fmt, g).values())
        if best is None or tot < best[1]:
            best = (n, tot)
    if best is None:
        raise ValueError("no block size fits the storage budget")
    return best[0]


def measure_sweep(shape=(4096, 4096)):
    """The sweep on the GPU: {(sigma, N, fmt): {'elem', 'max', 'zero'}} measured by the fused
    quantize + error-reduction pass on bf16 N(0, sigma^2) tensors (one grouped launch per point
    over the five sigma tensors)."""
    import fp4_microscaling_tensor_b200 as mx
    from fp4_microscaling_tensor_b200 import inputs
    xs = [inputs.workload2(k, shape=shape, device="cuda") for k in range(len(SIGMAS))]
    out = {}
    for n in BLOCKS:
        for fmt in (E4M3, UE5M3):
            _, _, st = mx.quantize_with_stats_group(xs, n, fmt)
            for k, s in enumerate(st):
                d = s.to_dict()
                out[(SIGMAS[k], n, fmt)] = {"elem": d["mse_elem"], "max": d["mse_max"],
                                            "zero": d["mse_zero"]}
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--measure", action="store_true", help="also measure the sweep on the GPU")
    args = ap.parse_args(argv)
    meas = measure_sweep() if args.measure else None
    hdr = "| sigma | N | fmt | model elem | model max | model zero | model total |"
    if meas:
        hdr += " measured elem | measured max | measured zero | total rel. diff |"
    print(hdr)
    print("|" + "---|" * (hdr.count("|") - 1))
    for s in SIGMAS:
        for n in BLOCKS:
            for fmt in (E4M3, UE5M3):
                m = model(s, n, fmt)
                tot = sum(m.values())
                row = (f"| {s} | {n} | {'E4M3' if fmt == E4M3 else 'UE5M3'} | {m['elem']:.4e} | "
                       f"{m['max']:.4e} | {m['zero']:.4e} | {tot:.4e} |")
                if meas:
                    e = meas[(s, n, fmt)]
                    et = sum(e.values())
                    row += (f" {e['elem']:.4e} | {e['max']:.4e} | {e['zero']:.4e} | "
                            f"{(et - tot) / tot:+.2e} |")
                print(row)
    return 0


if __name__ == "__main__":
    sys.exit(main())
