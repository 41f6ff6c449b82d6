"""Pins for the oracle's fixed codebook (Lloyd-Max quantiser of N(0,1))."""
import math
import struct

import numpy as np
import pytest
from scipy import integrate, stats

from oracle.codebook import distortion, lloyd_max_gaussian
from synth.workloads import codebook


def test_two_levels_closed_form():
    # 2-level optimum: +-E|X| = +-sqrt(2/pi), distortion 1 - 2/pi
    c = lloyd_max_gaussian(2)
    assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-12
    assert c[0] == -c[1]
    assert abs(distortion(c) - (1 - 2 / math.pi)) < 1e-12


def test_four_levels_match_printed_values():
    # the workload description prints the 2-bit codebook as +-0.4528, +-1.5104
    c = lloyd_max_gaussian(4)
    assert np.allclose(c, [-1.5104, -0.4528, 0.4528, 1.5104], atol=5e-5)
    # Max (1960), "Quantizing for minimum distortion", Table I: N=4 MSE 0.1175
    assert abs(distortion(c) - 0.1175) < 1e-4


def test_sixteen_levels_match_textbook():
    # Max (1960), Table I, N=16 output levels (positive half)
    want = [0.1284, 0.3881, 0.6568, 0.9424, 1.256, 1.618, 2.069, 2.733]
    c = lloyd_max_gaussian(16)
    assert np.allclose(c[8:], want, atol=1e-3)
    assert all(c[j] == -c[15 - j] for j in range(16))


@pytest.mark.parametrize("L", [4, 16])
def test_centroid_condition_by_quadrature(L):
    # each level is the conditional mean of its cell (thresholds at midpoints),
    # checked with numerical integration instead of the closed form
    c = lloyd_max_gaussian(L)
    thr = [-np.inf] + [(c[j] + c[j + 1]) / 2 for j in range(L - 1)] + [np.inf]
    for j in range(L):
        a, b = thr[j], thr[j + 1]
        num = integrate.quad(lambda x: x * stats.norm.pdf(x), a, b, epsabs=1e-14)[0]
        den = stats.norm.cdf(b) - stats.norm.cdf(a)
        assert abs(num / den - c[j]) < 1e-9


@pytest.mark.parametrize("L", [4, 16])
def test_distortion_is_local_minimum(L):
    c = np.array(lloyd_max_gaussian(L))
    d0 = distortion(c)
    rng = np.random.default_rng(1)
    for _ in range(20):
        eps = rng.normal(size=L) * 1e-3
        assert distortion(np.sort(c + eps)) > d0


def test_golden_file_is_fp32_of_oracle():
    for bits in (2, 4):
        L = 1 << bits
        ref = np.array(lloyd_max_gaussian(L), dtype=np.float32)
        got = codebook(bits)
        assert got.dtype == np.float32
        assert [struct.pack("<f", x) for x in got] == [struct.pack("<f", x) for x in ref]
