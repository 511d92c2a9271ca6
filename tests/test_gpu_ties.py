"""Rounding ties, boundary hits and saturation through the CUDA path (C ABI),
bit-exact against the oracle.

Random data almost never lands a value exactly on a rounding tie, so these rows
are planted in the rotated domain.  With Hadamard blocks of 256 the
normalisation 1/sqrt(256) = 1/16 is exact, so for a wanted rotated row y the
input v = H y / 16 (H the unnormalised Sylvester matrix, H H = 256 I) and
x = D P^T v reproduce y exactly in FP32, as long as every entry of v is a BF16
value (checked).  Covered: INT4 ties y * inv = k + 1/2 (TR-DQ section 3.1,
Eq. 1: round to nearest, ties read as ties-to-even) on activations and on
128-wide weight groups; NVFP4 (DiRotQ abstract) E2M1 ties after block scaling,
an E4M3-subnormal block scale, an E4M3 block-scale tie and a block scale
pushed to 448 by the rounded per-token multiplier; codebook codes
(OrbitQuant abstract) of values exactly on, or one ulp from, a boundary, found
by searching seeded rows with the oracle."""
import math

import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq
from tests import _harness as H

torch = pytest.importorskip("torch")

F32 = np.float32


def sylvester(n):
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def plant(y_rows, sign, perm, block=256):
    """BF16 bits of rows x whose rotation (signs, permutation, block FWHT,
    1/sqrt(block)) is exactly y_rows."""
    assert block == 256
    Hb = sylvester(block)
    M, K = y_rows.shape
    v = np.zeros((M, K))
    for b0 in range(0, K, block):
        v[:, b0:b0 + block] = y_rows[:, b0:b0 + block] @ Hb.T / 16.0
    bits = inputs.bf16_bits(v.astype(F32))
    assert np.array_equal(inputs.bf16_to_f32(bits).astype(np.float64), v), "v is not BF16-exact"
    x = np.zeros((M, K), dtype=np.uint16)
    xs = np.empty((M, K))
    xs[:, perm] = v * sign[perm][None, :]
    x = inputs.bf16_bits(xs.astype(F32))
    # the oracle's own rotation must give back y exactly
    y = orc.rotate(inputs.bf16_to_f32(x), sign, perm, block)
    assert np.array_equal(y.astype(np.float64), y_rows), "planted rows do not rotate back exactly"
    return x


def run_quant(fmt, X, block, weight=False, boundaries=None):
    K = X.shape[1]
    sign, perm, rot = rq.rq_make_rotation(K, block, 0)
    rot_t = torch.from_numpy(rot).cuda()
    g = H.gpu_quantize(fmt, X, block, rot_t, boundaries, None, weight=weight)
    o_sign, o_perm = orc.make_rotation(K, block, 0)
    o = orc.rotate_quantize(inputs.bf16_to_f32(X), fmt, block, o_sign, o_perm, boundaries, weight_rows=weight)
    H.assert_quant_equal(g, o, f"fmt {fmt}")
    return g, o


@pytest.mark.gpu
@pytest.mark.parametrize("weight", [False, True])
def test_int4_ties(weight):
    K = 512
    sign, perm = orc.make_rotation(K, 256, 0)
    ties = [7, 0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 3.5, -3.5, 4.5, -4.5, 5.5, -5.5, 6.5, -6.5]
    rows = []
    for scale in (1.0, 2.0 ** -4, 4.0):
        y = np.zeros(K)
        # one tie pattern per 128-wide group (a weight group gets its own amax)
        for g0 in range(0, K, 128):
            y[g0:g0 + len(ties)] = np.array(ties) * scale
        rows.append(y)
    y = np.array(rows)
    X = plant(y, sign, perm)
    g, o = run_quant(rq.INT4, X, 256, weight=weight)
    q = o["q"].astype(int)
    # amax 7 * scale: inv = 1/scale exactly, so y * inv = +-(k + 1/2) -> even
    want = [7, 0, 0, 2, -2, 2, -2, 4, -4, 4, -4, 6, -6, 6, -6]
    for r in range(3):
        for g0 in range(0, K, 128):
            assert list(q[r, g0:g0 + len(want)]) == want


@pytest.mark.gpu
def test_nvfp4_ties_subnormal_scale_and_saturation():
    K = 512
    sign, perm = orc.make_rotation(K, 256, 0)
    blocks = [
        # E2M1 ties after a block scale of 2 (E4M3 0x40)
        ([12, 0.5, 1.5, 2.5, 3.5, 5, 7, 10, -0.5, -1.5, -2.5, -3.5, -5, -7, -10, 0], 0x40,
         [7, 0, 2, 2, 4, 4, 6, 6, 8, 10, 10, 12, 12, 14, 14, 0]),
        # block scale 2^-8, an E4M3 subnormal (0x02)
        ([0.0234375, 0.001953125, -0.00390625, 0.0029296875] + [0] * 12, 0x02, [7, 1, 10, 2] + [0] * 12),
        # block scale 18.75 / 6 = 3.125: halfway between 3.0 and 3.25 -> 3.0 (0x44)
        ([18.75, 9, -4.5, 0.75] + [0] * 12, 0x44, [7, 5, 11, 0] + [0] * 12),
    ]
    rows = []
    for vals, _, _ in blocks:
        y = np.zeros(K)
        # u = y * 2688 / amax with amax 10.5: the multiplier is exactly 256
        y[:16] = np.array(vals) / 256.0
        y[256] = 10.5
        rows.append(y)
    y = np.zeros(K)
    y[0] = 4.875           # 4.875 * fp32(2688 / 4.875) rounds to 2688.0002: block scale 448
    rows.append(y)
    X = plant(np.array(rows), sign, perm)
    g, o = run_quant(rq.NVFP4, X, 256)
    sb, q = o["block_scale"], o["q"]
    for r, (_, want_sb, want_q) in enumerate(blocks):
        assert sb[r, 0] == want_sb and list(q[r, :16]) == want_q
        assert sb[r, 16] == 0x7E and q[r, 256] == 7        # the 2688 anchor
    assert sb[3, 0] == 0x7E and q[3, 0] == 7 and not q[3, 1:].any()


def boundary_rows(w, boundaries, n_rows=None, want=24):
    """Seeded rows of the workload's recipe whose normalised rotated values hit
    a codebook boundary exactly or within one ulp (searched with the oracle)."""
    K, b = w.K, w.block
    n_rows = n_rows or (6 << 20) // K
    sign, perm = orc.make_rotation(K, b, 0)
    X = inputs.activations(w, M=n_rows, token_seed=977)
    y = orc.rotate(inputs.bf16_to_f32(X), sign, perm, b)
    nrm = np.sqrt(orc.sum_squares(y, b)).astype(F32)
    u = (y * (F32(math.sqrt(K)) / nrm).astype(F32)[:, None]).astype(F32)
    bnd = np.asarray(boundaries, F32)
    near = np.zeros(n_rows, dtype=bool)
    exact = np.zeros(n_rows, dtype=bool)
    for t in bnd:
        lo, hi = np.nextafter(t, F32(-np.inf)), np.nextafter(t, F32(np.inf))
        exact |= np.any(u == t, axis=1)
        near |= np.any((u >= lo) & (u <= hi), axis=1)
    idx = np.concatenate([np.nonzero(exact)[0], np.nonzero(near & ~exact)[0]])[:want]
    return X[idx], int(exact.sum()), int(near.sum())


@pytest.mark.gpu
@pytest.mark.parametrize("name,levels", [("c5", 16), ("c3", 16)])
def test_codebook_boundary_hits(name, levels):
    w = inputs.WORKLOADS[name]
    cb = rq.rq_make_codebook(w.K, levels)
    X, n_exact, n_near = boundary_rows(w, cb["boundaries_f32"])
    assert n_exact >= 1 and len(X) >= 8, (n_exact, n_near)
    run_quant(rq.LM16, X, w.block, boundaries=cb["boundaries_f32"])


@pytest.mark.gpu
def test_codebook_boundary_hits_weights_lm4():
    w = inputs.WORKLOADS["c5"]
    cb = rq.rq_make_codebook(w.K, 4)
    X, n_exact, n_near = boundary_rows(w, cb["boundaries_f32"])
    assert n_near >= 1 and len(X) >= 1
    run_quant(rq.LM4, X, w.block, weight=True, boundaries=cb["boundaries_f32"])
