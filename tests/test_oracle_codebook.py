"""Pins for the oracle's Lloyd-Max codebook (CPU only).

OrbitQuant abstract: after the RPBH rotation every coordinate follows one known
marginal, and one Lloyd-Max codebook for it serves every input of a given
dimension.  Lloyd-Max optimality fixes two conditions that these tests check
against direct numerical integration of the density (independent of the
oracle's closed forms), plus the Gaussian limit (Max 1960).
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import rq_oracle as orc


def density(K):
    logc = orc.sphere_marginal_logc(K)
    a = (K - 3) / 2.0
    return lambda u: math.exp(logc + a * math.log1p(-u * u / K)) if u * u < K else 0.0


def quad(f, lo, hi):
    """Adaptive quadrature, split at +-4 and +-10 so the peak and the tails are
    resolved separately."""
    cuts = [lo] + [c for c in (-10.0, -4.0, 0.0, 4.0, 10.0) if lo < c < hi] + [hi]
    return sum(integrate.quad(f, a, b, epsabs=1e-16, epsrel=1e-13, limit=400)[0]
               for a, b in zip(cuts[:-1], cuts[1:]))


@pytest.mark.parametrize("K", [1152, 1536, 3072, 12288])
def test_density_normalised(K):
    f = density(K)
    L = min(math.sqrt(K), 40.0)
    assert abs(quad(f, -L, L) - 1.0) < 1e-12
    assert abs(quad(lambda u: u * u * f(u), -L, L) - 1.0) < 1e-10   # E[U^2] = 1


@pytest.mark.parametrize("K,levels", [(1152, 16), (3072, 16), (1536, 16), (1536, 4), (12288, 16)])
def test_lloyd_max_fixed_point(K, levels):
    cent, bnd = orc.lloyd_max(K, levels)
    assert len(cent) == levels and len(bnd) == levels - 1
    assert np.all(np.diff(cent) > 0) and np.all(np.diff(bnd) > 0)
    assert np.allclose(cent, -cent[::-1], atol=0) and bnd[levels // 2 - 1] == 0.0
    # boundaries are midpoints
    assert np.allclose(bnd, (cent[:-1] + cent[1:]) / 2, rtol=0, atol=1e-15)
    # centroids are conditional means (direct quadrature of the density)
    f = density(K)
    L = min(math.sqrt(K), 40.0)
    edges = [-L] + list(bnd) + [L]
    for i in range(levels):
        lo, hi = edges[i], edges[i + 1]
        m0 = quad(f, lo, hi)
        m1 = quad(lambda u: u * f(u), lo, hi)
        assert abs(m1 / m0 - cent[i]) < 1e-10, (i, m1 / m0, cent[i])


def gaussian_lloyd(levels, iters=20000):
    """Independent Gaussian Lloyd-Max (scipy.stats.norm), for the large-K limit."""
    h = levels // 2
    c = np.arange(h) * 3.0 / h + 1.5 / h
    for _ in range(iters):
        b = np.concatenate([[0.0], (c[:-1] + c[1:]) / 2, [np.inf]])
        mass = stats.norm.cdf(b[1:]) - stats.norm.cdf(b[:-1])
        c = (stats.norm.pdf(b[:-1]) - stats.norm.pdf(b[1:])) / mass
    return np.concatenate([-c[::-1], c])


def test_gaussian_limit_textbook_values():
    # Max (1960), 4-level Gaussian quantizer: outputs +-0.4528, +-1.510, threshold 0.9816
    cent, bnd = orc.lloyd_max(10 ** 6, 4)
    assert np.allclose(cent, [-1.510, -0.4528, 0.4528, 1.510], atol=6e-4)
    assert abs(bnd[2] - 0.9816) < 6e-4
    g16 = gaussian_lloyd(16)
    c16, _ = orc.lloyd_max(10 ** 6, 16)
    assert np.allclose(c16, g16, atol=5e-5)


def test_codebook_mse_gaussian_4level():
    """MSE of the 4-level Gaussian Lloyd-Max quantizer is 0.1175 (Max 1960)."""
    c = gaussian_lloyd(4)
    b = np.concatenate([[-np.inf], (c[:-1] + c[1:]) / 2, [np.inf]])
    mse = sum(integrate.quad(lambda u: (u - c[i]) ** 2 * stats.norm.pdf(u), b[i], b[i + 1])[0]
              for i in range(4))
    assert abs(mse - 0.1175) < 2e-4
    cent, _ = orc.lloyd_max(10 ** 6, 4)
    assert np.allclose(cent, c, atol=5e-5)


def test_tables():
    bf32, ce4 = orc.codebook_tables(3072, 16)
    assert bf32.dtype == np.float32 and ce4.dtype == np.uint8 and len(bf32) == 15 and len(ce4) == 16
    vals = orc.e4m3_decode(ce4)
    cent, _ = orc.lloyd_max(3072, 16)
    assert np.all(np.abs(vals - cent) <= np.abs(cent) * 2.0 ** -4 + 1e-12)   # e4m3: 3 mantissa bits
