"""Numpy model of the golden-label kernel's fp32 total Z and its error bound (csrc/golden.cuh,
k_golden_nucleus fast path) against the exact sum, on the CPU.

The kernel sums e = 2^((z - m) log2 e) in fp32, per thread over its own entries (16-byte vectors
v = t, t + 256, t + 512, ... of the row, four entries each, then at most one lone entry), and adds
the 256 per-thread sums in double.  It certifies the nucleus crossing against Z32 +- err with

    err = 1.01 Z32 (2^-22 + 3 * 104 * 2^-24 + (S / 256 + 5) 2^-24) + S 2^-126
          + 2 Z32 (S / 256 + 64) 2^-53.

The model evaluates the same sums in the same order with numpy's fp32 arithmetic (each operation
rounded to nearest; numpy's fp32 exp2 stands in for the device's, both within 2 ulp) and checks
|Z32 - Z| <= err, Z the exactly rounded sum of exp(z - m) (math.fsum over float64 terms), on rows
built to stress each term: large |z - m| (the argument rounding), long rows (the per-thread sums),
subnormal terms, all-equal rows and rows with one dominant entry.
"""
import math

import numpy as np
import pytest

THREADS = 256
LOG2E = np.float32(1.4426950408889634)


def z32_model(z):
    """(Z32, err) as the kernel computes them for an aligned row z (float32)."""
    S = z.size
    m = np.float32(z.max())
    nvec = S // 4
    tail0 = 4 * nvec
    zf = np.zeros(THREADS, dtype=np.float32)
    for t in range(THREADS):
        acc = np.float32(0.0)
        for v in range(t, nvec, THREADS):
            for x in z[4 * v: 4 * v + 4]:
                a = np.float32(np.float32(x - m) * LOG2E)
                acc = np.float32(acc + np.exp2(a))
        zf[t] = acc
    for i, s in enumerate(range(tail0, S)):  # lone entries: threads 0, 1, ...
        a = np.float32(np.float32(z[s] - m) * LOG2E)
        zf[i] = np.float32(zf[i] + np.exp2(a))
    Z32 = float(np.sum(zf.astype(np.float64)))
    err = (1.01 * Z32 * (2.0 ** -22 + 3.0 * 104.0 * 2.0 ** -24 + (S / THREADS + 5.0) * 2.0 ** -24)
           + S * 2.0 ** -126 + 2.0 * Z32 * (S / THREADS + 64.0) * 2.0 ** -53)
    return Z32, err


def z_exact(z):
    m = float(z.max())
    return math.fsum(math.exp(float(x) - m) for x in z)


def rows():
    rng = np.random.default_rng(11)
    yield "normal_32k", rng.standard_normal(32768).astype(np.float32)
    peaks = rng.standard_normal(32768).astype(np.float32)
    peaks[rng.integers(0, 32768, 400)] += 6.0
    yield "planted_peaks", peaks
    yield "wide_range", rng.uniform(-100.0, 0.0, 8192).astype(np.float32)
    yield "subnormal_terms", np.concatenate([np.zeros(4, np.float32),
                                             rng.uniform(-103.0, -87.0, 4092).astype(np.float32)])
    yield "all_equal", np.full(5000, 3.25, dtype=np.float32)
    dom = np.full(9999, -40.0, dtype=np.float32)
    dom[1234] = 0.0
    yield "one_dominant_ragged", dom
    yield "tiny_ragged", rng.standard_normal(7).astype(np.float32)
    # the worst case of the per-thread sums: the thread holding the maximum adds 127 terms of
    # 2^-24, each of which rounds away against its running sum of 1
    lost = np.full(32768, np.float32(-24.0 * math.log(2.0)), dtype=np.float32)
    lost[0] = 0.0
    yield "rounding_lost_terms", lost


@pytest.mark.parametrize("name,z", list(rows()), ids=[n for n, _ in rows()])
def test_fp32_total_within_its_bound(name, z):
    Z32, err = z32_model(z)
    Z = z_exact(z)
    assert abs(Z32 - Z) <= err, (name, Z32, Z, err)
    # the bound is not vacuous: a few parts in 10^5 of Z at most on these rows
    assert err <= 1e-4 * Z, (name, err / Z)
