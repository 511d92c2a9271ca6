"""Pins for the oracle's TR-DQ pieces (CPU): the zigzag permutation and the
double block rotation (TR-DQ: Time-Rotation Diffusion Quantization, section
3.2, Eq. 9), asymmetric per-token INT4 (section 3.1, Eq. 1-3) and the 8-bit
per-token / per-channel settings."""
import math

import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs

F32 = np.float32


def test_zigzag_hand_dealt():
    # K = 8 channels, blocks of 2 -> 4 blocks; ranked: 4 (9), 6 (7), 1 (5),
    # 2 (3), 5 (1), 7 (0.3), 3 (0.2), 0 (0.1).  The first pass deals blocks
    # 0..3 their first slot, the second pass blocks 3..0 their second slot.
    mag = [0.1, 5, 3, 0.2, 9, 1, 7, 0.3]
    assert list(orc.zigzag_permutation(mag, 2)) == [4, 0, 6, 3, 1, 7, 2, 5]
    # equal magnitudes rank by channel index
    assert list(orc.zigzag_permutation([1, 1, 1, 1], 2)) == [0, 3, 1, 2]


def test_zigzag_bijection_and_balance():
    rng = np.random.default_rng(3)
    K, b = 1536, 128
    mag = rng.lognormal(0, 2, K)
    p = orc.zigzag_permutation(mag, b)
    assert sorted(p) == list(range(K))
    rank = np.empty(K, int)
    rank[np.argsort(-mag, kind="stable")] = np.arange(K)
    per_block = rank[p].reshape(K // b, b).sum(axis=1)
    # an even number of rounds gives every block the same rank sum
    assert np.all(per_block == per_block[0])
    # the largest channel goes to block 0, the next to block 1
    assert p[0] == np.argmax(mag) and rank[p[b]] == 1


def _dense_rotation(K, sign, perm, b):
    Hb = np.ones((1, 1))
    while Hb.shape[0] < b:
        Hb = np.block([[Hb, Hb], [Hb, -Hb]])
    H = np.kron(np.eye(K // b), Hb / math.sqrt(b))
    P = np.zeros((K, K))
    P[np.arange(K), perm] = 1.0
    D = np.diag(sign.astype(np.float64))
    return H, P, D


def test_double_rotation_is_the_matrix_product():
    K, b = 64, 16
    sign, _ = orc.make_rotation(K, b, 5)
    zz = orc.zigzag_permutation(np.random.default_rng(1).random(K), b)
    H, P, D = _dense_rotation(K, sign, zz, b)
    R = H @ P @ H @ D
    x = np.random.default_rng(2).standard_normal((5, K))
    assert np.allclose(orc.rotate_double(x, sign, zz, b), x @ R.T, atol=1e-12)
    assert np.allclose(R @ R.T, np.eye(K), atol=1e-12)
    # folded into the weights the rotation cancels inside the layer (Eq. 9)
    W = np.random.default_rng(4).standard_normal((7, K))
    xr = orc.rotate_double(x, sign, zz, b)
    wr = orc.rotate_double(W, sign, zz, b)
    assert np.allclose(xr @ wr.T, x @ W.T, rtol=1e-12, atol=1e-10)


def test_asym_int4_hand_rows():
    y = np.array([[-1.0, 0.0, 0.5, 2.0],
                  [0.0625, 1.9375, 1.0, 0.3125]], dtype=F32)
    nib, s, zp = orc.quant_int4_asym(y)
    # row 0: range 3, inv 5, z = round(-5) = -5; y * inv = -5, 0, 2.5 (tie -> 2), 10
    assert list(nib[0]) == [-8, -3, -1, 7] and zp[0] == 3 and s[0] == F32(F32(3) / F32(15))
    # row 1: range 1.875, inv 8 exactly, min * inv = 0.5 -> z = 0 (tie to even);
    # max * inv = 15.5 -> 16 -> clamped to 15; 0.3125 * 8 = 2.5 -> 2
    assert list(nib[1]) == [-8 + 0, 7, -8 + 8, -8 + 2] and zp[1] == 8
    assert s[1] == F32(0.125)
    nib, s, zp = orc.quant_int4_asym(np.zeros((1, 4), F32))
    assert list(nib[0]) == [-8] * 4 and s[0] == 0 and zp[0] == 8


def test_asym_int4_error_bound():
    rng = np.random.default_rng(7)
    y = (rng.standard_normal((40, 256)) * rng.uniform(0.1, 10, (40, 1)) + rng.uniform(-3, 3, (40, 1))).astype(F32)
    nib, s, zp = orc.quant_int4_asym(y)
    xr = s[:, None].astype(np.float64) * (nib.astype(np.float64) + zp[:, None])
    assert np.all(np.abs(xr - y) <= s[:, None] * (1.0 + 1e-5))
    assert np.all(nib.min(axis=1) == -8) and np.all(nib.max(axis=1) == 7)


def test_asym_gemm_is_the_dequantized_product():
    rng = np.random.default_rng(8)
    y = rng.standard_normal((3, 256)).astype(F32) + F32(0.7)
    nib, s, zp = orc.quant_int4_asym(y)
    qw = rng.integers(-7, 8, (4, 256)).astype(np.int8)
    sw = rng.uniform(0.1, 1, (2, 4)).astype(F32)
    Y = orc.reference_gemm(orc.INT4A, orc.INT4, nib, s, qw, sw, a_zp=zp)
    A = s[:, None].astype(np.float64) * (nib + zp[:, None])
    B = qw.astype(np.float64) * np.repeat(sw.T.astype(np.float64), 128, axis=1)
    assert np.allclose(Y, A @ B.T, rtol=1e-12)


def test_int8_hand_cases_and_bound():
    # amax 127 -> inv 1 exactly: ties at .5 go to even, the maximum lands on 127
    y = np.array([[127.0, 0.5, -0.5, 1.5, -2.5, 126.5, -126.5, 3.0]], dtype=F32)
    q, s = orc.quant_int8(y)
    assert list(q[0]) == [127, 0, 0, 2, -2, 126, -126, 3] and s[0] == F32(1.0)
    q, s = orc.quant_int8(np.zeros((1, 8), F32))
    assert s[0] == 0 and not q.any()
    rng = np.random.default_rng(9)
    y = (rng.standard_normal((30, 256)) * rng.uniform(0.1, 10, (30, 1))).astype(F32)
    q, s = orc.quant_int8(y)
    assert np.all(np.abs(q * s[:, None].astype(np.float64) - y) <= s[:, None] * 0.5 * (1 + 1e-6))
    assert np.all(np.max(np.abs(q.astype(int)), axis=1) == 127)
    # W4A8: the reference GEMM multiplies the integer codes with the grouped weights
    qw = rng.integers(-7, 8, (5, 256)).astype(np.int8)
    sw = rng.uniform(0.1, 1, (2, 5)).astype(F32)
    Y = orc.reference_gemm(orc.INT8, orc.INT4, q, s, qw, sw)
    B = qw.astype(np.float64) * np.repeat(sw.T.astype(np.float64), 128, axis=1)
    assert np.allclose(Y, (q * s[:, None].astype(np.float64)) @ B.T, rtol=1e-12)


def test_w8a8_weight_rows_per_channel():
    # W8A8 (TR-DQ section 3.1: per-channel weights): one scale per rotated
    # weight row, amax/127, and the layer tracks x W^T closer than W4A8 does
    w = inputs.WORKLOADS["c1"]
    sign, perm = orc.make_rotation(w.K, w.block, 0)
    X = inputs.bf16_to_f32(inputs.activations(w, M=64))
    W = inputs.bf16_to_f32(inputs.weights(w, N=96))
    ow = orc.rotate_quantize(W, orc.INT8, w.block, sign, perm, weight_rows=True)
    yw = orc.rotate(W, sign, perm, w.block)
    assert ow["scale"].shape == (96,)
    assert np.array_equal(ow["scale"], (np.max(np.abs(yw), axis=1) / np.float32(127)).astype(np.float32))
    assert np.all(np.abs(ow["q"].astype(np.float64) * ow["scale"][:, None] - yw) <= ow["scale"][:, None] * 0.5 * (1 + 1e-6))
    oa = orc.rotate_quantize(X, orc.INT8, w.block, sign, perm)
    o4 = orc.rotate_quantize(W, orc.INT4, w.block, sign, perm, weight_rows=True)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    e8 = np.linalg.norm(orc.reference_gemm(orc.INT8, orc.INT8, oa["q"], oa["scale"], ow["q"], ow["scale"]) - ref)
    e4 = np.linalg.norm(orc.reference_gemm(orc.INT8, orc.INT4, oa["q"], oa["scale"], o4["q"], o4["scale"]) - ref)
    assert e8 < 0.5 * e4
