"""Error bounds the tensor-core path relies on, checked by emulating its
bf16 / fp32 operations in numpy (CPU only).

* Pass 2's fast path replaces p / (1 - p) by p t(p) for p < 2^-4, t the
  minimax quadratic of 1 / (1 - p) in relative error on [0, 2^-4]: relative
  error <= 1 / T3(31) = 8.4e-6 (ratio^2: 1.7e-5).  The kernel's three
  coefficients are read from its source and rebuilt here from numpy's
  Chebyshev polynomials.
* Pass 1 stores P in [0, 256] as P_hi = P truncated to bf16 plus
  P_lo = bf16_rn(P - P_hi): P to 2^-16 relative.
* The combine stores -2A as bf16_rn hi + bf16_rn lo: to 2^-16 relative per
  component.
* Pass 2 drops A_lo when ||A||^2 <= 8e-4 ||v||^2 everywhere: the squared
  distance then moves by at most 2^-7 rho / (1 - rho)^2 <= 2.4e-4 relative.
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def bf16_trunc(x):
    u = np.asarray(x, np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def bf16_rn(x):
    """Round-to-nearest-even to bf16 (finite inputs)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def test_bf16_rounding_emulation():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties to even
    x = np.float32(1.0 + 2.0 ** -8)
    assert bf16_rn(x) == np.float32(1.0)
    assert bf16_rn(np.float32(1.0 + 3 * 2.0 ** -8)) == np.float32(1.0 + 2.0 ** -6)
    assert bf16_trunc(np.float32(1.0 + 3 * 2.0 ** -8)) == np.float32(1.0 + 2.0 ** -7)


def _kernel_ratio_coefficients():
    src = open(os.path.join(ROOT, "kv_cache_eviction_scores_b200", "csrc", "tc_common.cuh")).read()
    m = re.search(r"constexpr float kT0 = ([0-9.]+)f, kT1 = ([0-9.]+)f, kT2 = ([0-9.]+)f;", src)
    assert m, "the fast ratio's coefficients are not in tc_common.cuh"
    return np.array([np.float32(float(x)) for x in m.groups()], np.float32)


def test_fast_path_ratio_coefficients_are_the_chebyshev_construction():
    # t(p) (1 - p) = 1 - T3(32 p - 1) / T3(31): numpy's T3 on the domain
    # [0, 2^-4] is T3(32 p - 1), and p = 1 maps to 31
    T3 = np.polynomial.Chebyshev.basis(3, domain=[0.0, 2.0 ** -4])
    assert T3(1.0) == 119071.0
    num = (1 - T3 / T3(1.0)).convert(kind=np.polynomial.Polynomial)
    t, rem = divmod(num, np.polynomial.Polynomial([1.0, -1.0]))
    assert t.degree() == 2 and np.abs(rem.coef).max() < 1e-9
    assert np.array_equal(t.coef.astype(np.float32), _kernel_ratio_coefficients())


def test_fast_path_ratio_error():
    c = _kernel_ratio_coefficients().astype(np.float64)
    p = np.linspace(1e-9, 2.0 ** -4, 400001)
    ratio = p * (c[0] + p * (c[1] + p * c[2]))
    exact = p / (1 - p)
    rel = np.abs(ratio - exact) / exact
    assert rel.max() <= 8.5e-6
    # equioscillation: at the four extrema of T3(32 p - 1) on [0, 2^-4] the
    # error alternates in sign at (within the coefficients' fp32 rounding)
    # the bound 1 / 119071
    pk = (1 + np.cos(np.arange(4) * np.pi / 3)) / 32
    e = (c[0] + pk * (c[1] + pk * c[2])) * (1 - pk) - 1
    assert np.all(np.sign(e[:-1]) != np.sign(e[1:]))
    assert np.allclose(np.abs(e), 1 / 119071, rtol=0.02)
    # the Taylor quadratic, p (1 + p + p^2), is off by p^3 relative: 2.4e-4 at 2^-4
    assert rel.max() < 0.1 * (2.0 ** -4) ** 3


def test_probability_hi_lo_split():
    rng = np.random.default_rng(0)
    P = np.concatenate([rng.uniform(0, 256, 200000), 2.0 ** rng.uniform(-40, 8, 200000)])
    P = P.astype(np.float32)
    hi = bf16_trunc(P)
    lo = bf16_rn(P - hi)  # P - hi is exact in fp32
    err = np.abs((hi.astype(np.float64) + lo) - P) / P
    assert err.max() <= 2.0 ** -16
    assert (hi <= P).all() and (np.abs(P - hi) < 2.0 ** -7 * P + 1e-45).all()


def test_output_hi_lo_split():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(400000) * 10.0 ** rng.uniform(-6, 3, 400000)).astype(np.float32)
    hi = bf16_rn(x)
    lo = bf16_rn(x - hi)
    err = np.abs((hi.astype(np.float64) + lo) - x) / np.abs(x)
    assert err.max() <= 2.0 ** -16


def test_dropping_the_low_part_bound():
    rho = np.sqrt(8e-4)
    assert 2.0 ** -7 * rho / (1 - rho) ** 2 <= 2.4e-4
    # worst case realised: components of -2A rounded to bf16 by up to 2^-8
    # relative, v aligned to maximise the moved inner product
    rng = np.random.default_rng(2)
    worst = 0.0
    for _ in range(200):
        v = rng.standard_normal(128)
        a = rng.standard_normal(128)
        a *= rho * np.linalg.norm(v) / np.linalg.norm(a)
        x = (-2 * a).astype(np.float32)
        moved = abs((bf16_rn(x).astype(np.float64) - x) @ v)
        z = np.sum((a - v) ** 2)
        worst = max(worst, moved / z)
    assert worst <= 2.4e-4
