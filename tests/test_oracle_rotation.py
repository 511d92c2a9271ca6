"""Pins for the oracle's RPBH rotation (CPU only).

What the pages fix: the rotation is orthogonal and built as a randomized,
permuted block-Hadamard transform (OrbitQuant abstract; TR-DQ section 3.2,
Eq. 8), so folding it into the weights cancels it inside the layer (TR-DQ Eq. 9).
"""
import itertools
import math
import os

import numpy as np
import pytest

from oracle import rq_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sylvester(b):
    """Dense Sylvester Hadamard by the Kronecker recursion H_2n = [[H, H], [H, -H]]."""
    H = np.array([[1.0]])
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def test_splitmix64_published_outputs():
    lines = [l.split() for l in open(os.path.join(GOLDEN, "splitmix64.txt")) if not l.startswith("#")]
    seed = int(lines[0][1])
    want = [int(l[0]) for l in lines[1:]]
    g = orc.SplitMix64(seed)
    assert [g.next() for _ in want] == want


@pytest.mark.parametrize("K,b,seed", [(1152, 128, 0), (12288, 256, 0), (64, 16, 5)])
def test_rotation_tables(K, b, seed):
    sign, perm = orc.make_rotation(K, b, seed)
    assert sign.dtype == np.int8 and perm.dtype == np.int32
    assert set(np.unique(sign)) <= {-1, 1}
    assert np.array_equal(np.sort(perm), np.arange(K))
    s2, p2 = orc.make_rotation(K, b, seed)
    assert np.array_equal(sign, s2) and np.array_equal(perm, p2)
    s3, p3 = orc.make_rotation(K, b, seed + 1)
    assert not np.array_equal(perm, p3)
    # signs are balanced (binomial, 6 sigma)
    assert abs(int(sign.astype(int).sum())) < 6 * math.sqrt(K)


def test_fisher_yates_uniform_on_k4():
    counts = {}
    n = 4800
    for seed in range(n):
        _, p = orc.make_rotation(4, 2, seed)
        counts[tuple(p)] = counts.get(tuple(p), 0) + 1
    assert len(counts) == 24
    exp = n / 24
    chi2 = sum((c - exp) ** 2 / exp for c in counts.values())
    assert chi2 < 60  # 23 dof, p ~ 1e-4


def test_below_is_in_range_and_unbiased():
    g = orc.SplitMix64(3)
    draws = [g.below(3) for _ in range(30000)]
    assert set(draws) == {0, 1, 2}
    for v in range(3):
        assert abs(draws.count(v) - 10000) < 500


@pytest.mark.parametrize("b", [2, 4, 8, 16])
def test_fwht_matches_dense_hadamard(b):
    H = sylvester(b)
    assert np.array_equal(H @ H.T, b * np.eye(b))
    rng = np.random.default_rng(b)
    # integer inputs: exact
    xi = rng.integers(-50, 50, size=(7, 3 * b)).astype(np.float64)
    want = np.concatenate([xi[:, j * b:(j + 1) * b] @ H.T for j in range(3)], axis=1)
    assert np.array_equal(orc.fwht_blocks(xi, b), want)
    # float32 integers stay exact too
    assert np.array_equal(orc.fwht_blocks(xi.astype(np.float32), b), want.astype(np.float32))
    xr = rng.standard_normal((5, 2 * b))
    want = np.concatenate([xr[:, j * b:(j + 1) * b] @ H.T for j in range(2)], axis=1)
    assert np.allclose(orc.fwht_blocks(xr, b), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("K,b", [(64, 16), (256, 16), (1152, 128)])
def test_rotation_is_the_documented_product(K, b):
    """R = BlockDiag(H_b / sqrt b) . P . D with P[i, perm[i]] = 1, D = diag(sign)."""
    sign, perm = orc.make_rotation(K, b, 1)
    R = orc.rotation_matrix(K, sign, perm, b)
    Hb = sylvester(b) / math.sqrt(b)
    BD = np.kron(np.eye(K // b), Hb)
    P = np.zeros((K, K))
    P[np.arange(K), perm] = 1.0
    D = np.diag(sign.astype(np.float64))
    assert np.allclose(R, BD @ P @ D, rtol=0, atol=1e-14)
    assert np.allclose(R.T @ R, np.eye(K), rtol=0, atol=1e-12)


def test_rotation_preserves_norm_fp64():
    K, b = 3072, 128
    sign, perm = orc.make_rotation(K, b, 0)
    x = np.random.default_rng(0).standard_normal((9, K))
    y = orc.rotate(x, sign, perm, b)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


@pytest.mark.parametrize("K,b", [(1152, 128), (12288, 256)])
def test_rotation_cancels_inside_layer(K, b):
    """x R^T R W^T = x W^T (FP64, 1e-5 relative): the rotation folded into the
    weights cancels the one applied to the activations."""
    sign, perm = orc.make_rotation(K, b, 0)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, K))
    x[:, :4] *= 30
    W = rng.standard_normal((24, K)) * 0.02
    y_rot = orc.rotate(x, sign, perm, b) @ orc.rotate(W, sign, perm, b).T
    y = x @ W.T
    rel = np.linalg.norm(y_rot - y) / np.linalg.norm(y)
    assert rel < 1e-5
    assert rel < 1e-12  # in fact it holds to rounding


def test_fp32_rotation_tracks_fp64():
    K, b = 1152, 128
    sign, perm = orc.make_rotation(K, b, 0)
    x = np.random.default_rng(2).standard_normal((4, K)).astype(np.float32)
    y32 = orc.rotate(x, sign, perm, b)
    y64 = orc.rotate(x.astype(np.float64), sign, perm, b)
    assert y32.dtype == np.float32
    assert np.max(np.abs(y32 - y64)) < 1e-5 * np.max(np.abs(y64))


def test_bad_block_rejected():
    with pytest.raises(ValueError):
        orc.make_rotation(100, 48, 0)
    with pytest.raises(ValueError):
        orc.make_rotation(100, 64, 0)
