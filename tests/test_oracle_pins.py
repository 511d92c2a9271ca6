"""Pins for the parts of the oracle whose result is fixed by an operation order
or a rounding rule rather than by a closed form (CPU only).

* The DiRotQ low-rank branch (DiRotQ abstract: the PCA coefficients are kept at
  higher precision and the remaining components are quantized): the
  coefficients c = x U and the residual x - c U^T, against element-by-element
  float32 loops written separately from the oracle, on inputs where the
  plausible wrong orders and a missing BF16 rounding give other values.
* NVFP4 (DiRotQ abstract: NVFP4 on Blackwell): hand-worked rows whose block
  scales and codes follow from the OCP E4M3 / E2M1 definitions by hand.
"""
import math
import struct

import numpy as np

from oracle import rq_oracle as orc

F32 = np.float32


def bf16_round_independent(v: float) -> int:
    """BF16 bits of the FP32 value v, round to nearest, ties to even, from the
    two neighbouring BF16 values (not the oracle's integer trick)."""
    bits = struct.unpack("<I", struct.pack("<f", float(v)))[0]
    lo = bits >> 16                        # truncation toward zero
    hi = lo + 1
    lo_v = struct.unpack("<f", struct.pack("<I", lo << 16))[0]
    hi_v = struct.unpack("<f", struct.pack("<I", hi << 16))[0]
    d_lo, d_hi = abs(float(v) - lo_v), abs(hi_v - float(v))
    if d_lo < d_hi or (d_lo == d_hi and lo % 2 == 0):
        return lo
    return hi


def spread_bf16(rng, shape, lo_exp, hi_exp):
    """BF16-representable values N(0,1) x 2^e with e uniform in [lo_exp, hi_exp]."""
    v = rng.standard_normal(shape) * np.exp2(rng.integers(lo_exp, hi_exp + 1, shape))
    bits = np.vectorize(bf16_round_independent)(v.astype(F32))
    return (bits.astype(np.uint32) << 16).view(F32)


def loop_coefficients(x, U, chunk=128):
    """c[m, j]: per chunk of `chunk` channels a float32 running sum of the
    products in k order, then the chunk sums added in chunk order."""
    M, K = x.shape
    r = U.shape[1]
    out = np.zeros((M, r), F32)
    for m in range(M):
        for j in range(r):
            total = None
            for t in range(K // chunk):
                acc = F32(0.0)
                for k in range(t * chunk, (t + 1) * chunk):
                    acc = F32(acc + F32(x[m, k] * U[k, j]))
                total = acc if total is None else F32(total + acc)
            out[m, j] = total
    return out


def loop_sequential(x, U):
    return loop_coefficients(x, U, chunk=x.shape[1])


def loop_pairwise_chunks(x, U, chunk=128):
    M, K = x.shape
    out = np.zeros((M, U.shape[1]), F32)
    for m in range(M):
        for j in range(U.shape[1]):
            total = None
            for t in range(K // chunk):
                vals = [F32(x[m, k] * U[k, j]) for k in range(t * chunk, (t + 1) * chunk)]
                while len(vals) > 1:
                    vals = [F32(vals[i] + vals[i + 1]) for i in range(0, len(vals), 2)]
                total = vals[0] if total is None else F32(total + vals[0])
            out[m, j] = total
    return out


def _lowrank_inputs():
    rng = np.random.default_rng(2024)
    x = spread_bf16(rng, (3, 384), -8, 8)
    U = spread_bf16(rng, (384, 6), -6, 2)
    return x, U


def test_projection_order_is_the_chunked_sum():
    x, U = _lowrank_inputs()
    want = loop_coefficients(x, U)
    got = orc.project_coefficients(x, U)
    assert got.dtype == F32
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # each plausible alternative reading gives other values on these inputs
    alternatives = {
        "blas": (x @ U).astype(F32),
        "one sequential chain": loop_sequential(x, U),
        "pairwise tree per chunk": loop_pairwise_chunks(x, U),
        "64-wide chunks": loop_coefficients(x, U, chunk=64),
        "exact then rounded": (x.astype(np.float64) @ U.astype(np.float64)).astype(F32),
    }
    for name, alt in alternatives.items():
        assert not np.array_equal(alt.view(np.uint32), want.view(np.uint32)), name


def test_coefficients_are_rounded_to_bf16_and_the_residual_uses_them():
    x, U = _lowrank_inputs()
    sign, perm = orc.make_rotation(384, 128, 3)
    out = orc.rotate_quantize(x, orc.INT4, 128, sign, perm, U_f32=U)
    c32 = loop_coefficients(x, U)
    want_bits = np.vectorize(bf16_round_independent)(c32).astype(np.uint16)
    assert np.array_equal(out["coef"], want_bits)
    assert not np.array_equal(c32.view(np.uint32) >> 16, want_bits.astype(np.uint32))  # rounding, not truncation
    # the quantized codes are those of the residual with the BF16 coefficients
    cb = (want_bits.astype(np.uint32) << 16).view(F32)
    y = orc.rotate(loop_residual(x, cb, U), sign, perm, 128)
    q, s = orc.quant_int4(y)
    assert np.array_equal(out["q"], q) and np.array_equal(out["scale"], s[:, 0])
    y_unrounded = orc.rotate(loop_residual(x, c32, U), sign, perm, 128)
    assert not np.array_equal(orc.quant_int4(y_unrounded)[1][:, 0], s[:, 0])


def loop_residual(x, c, U):
    M, K = x.shape
    out = np.empty_like(x)
    for m in range(M):
        for k in range(K):
            v = F32(x[m, k])
            for j in range(U.shape[1]):
                v = F32(v - F32(c[m, j] * U[k, j]))
            out[m, k] = v
    return out


def test_residual_order():
    x, U = _lowrank_inputs()
    cb = (np.vectorize(bf16_round_independent)(loop_coefficients(x, U)).astype(np.uint32) << 16).view(F32)
    want = loop_residual(x, cb, U)
    got = orc.residual(x, cb, U)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    alternatives = {
        "blas": (x - cb @ U.T).astype(F32),
        "reverse j": loop_residual(x, cb[:, ::-1].copy(), U[:, ::-1].copy()),
        "exact then rounded": (x.astype(np.float64) - cb.astype(np.float64) @ U.astype(np.float64).T).astype(F32),
    }
    for name, alt in alternatives.items():
        assert not np.array_equal(alt.view(np.uint32), want.view(np.uint32)), name


# ---------------------------------------------------------------------- NVFP4
# Row 1 has amax 2688, so the per-token scale is exactly 1 and u = y.  Block by
# block (E4M3 values: 2.0 = 0x40, 448 = 0x7E, 2^-8 = subnormal 0x02, 3.0 = 0x44,
# 1.875 = 0x3F):
#  B0  max 12 -> 12/6 = 2.0 -> 0x40; 1/sb = 0.5, so u/2 lands on the E2M1
#      midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 -> ties to the even code.
#  B1  max 2688 -> 448 -> 0x7E; fp32(1/448) is 4.5e-8 high: 2688 -> 6.0000003
#      saturates to 6, 1344 -> 3, -896 -> -2, 672 -> 1.5, 112 -> exactly 0.25
#      (tie -> 0), 336 -> 0.75000006 (above the midpoint -> 1.0).
#  B2  max 0.0234375 = 6 * 2^-8 -> 2^-8, an E4M3 subnormal (0x02); 1/sb = 256:
#      codes of 6, 0.5, -1, 0.75 (tie -> 1.0).
#  B3  max 18.75 -> 3.125, halfway between 3.0 (mantissa 4) and 3.25 (mantissa
#      5) -> even -> 3.0 = 0x44; fp32(1/3): 18.75 -> 6.25 -> 6, 9 -> 3, -4.5 ->
#      -1.5, 0.75 -> exactly 0.25 (tie -> 0).
#  B4  max 11.25 -> 1.875 = 0x3F; fp32(1/1.875) is 4.5e-8 high, so u * (1/sb)
#      lands just above the midpoints that u / sb would hit exactly:
#      2.34375 -> 1.2500001 -> 1.5, 4.6875 -> 2.5000002 -> 3, 9.375 ->
#      5.0000005 -> 6, 11.25 -> 6.
#  B5  all zero -> block scale 0, codes 0.
# Row 2 has amax 4.875: inv = fp32(2688 / 4.875) and 4.875 * inv rounds to
# 2688.0002, so its block scale 448.00003 rounds to the largest E4M3 value 448
# (0x7E) and its code saturates at 6.
E2M1 = {0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def _code(v):
    return E2M1[abs(v)] | (8 if v < 0 or (v == 0 and math.copysign(1, v) < 0) else 0)


NVFP4_ROW1 = [
    ([12, 0.5, 1.5, 2.5, 3.5, 5, 7, 10, -0.5, -1.5, -2.5, -3.5, -5, -7, -10, 0], 0x40,
     [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -0.0, -1.0, -1.0, -2.0, -2.0, -4.0, -4.0, 0.0]),
    ([2688, 1344, -896, 672, 112, 336] + [0] * 10, 0x7E, [6.0, 3.0, -2.0, 1.5, 0.0, 1.0] + [0.0] * 10),
    ([0.0234375, 0.001953125, -0.00390625, 0.0029296875] + [0] * 12, 0x02, [6.0, 0.5, -1.0, 1.0] + [0.0] * 12),
    ([18.75, 9, -4.5, 0.75] + [0] * 12, 0x44, [6.0, 3.0, -1.5, 0.0] + [0.0] * 12),
    ([11.25, 2.34375, 4.6875, 9.375] + [0] * 12, 0x3F, [6.0, 1.5, 3.0, 6.0] + [0.0] * 12),
    ([0] * 16, 0x00, [0.0] * 16),
]


def test_nvfp4_hand_worked_rows():
    row1 = np.array([v for blk, _, _ in NVFP4_ROW1 for v in blk], dtype=F32)[None, :]
    row2 = np.zeros((1, 96), F32)
    row2[0, 0] = 4.875
    q, sb, s = orc.quant_nvfp4(np.concatenate([row1, row2]))
    assert list(sb[0]) == [b for _, b, _ in NVFP4_ROW1]
    assert list(q[0]) == [_code(v) for _, _, vals in NVFP4_ROW1 for v in vals]
    assert s[0] == F32(1.0)
    assert list(sb[1]) == [0x7E, 0, 0, 0, 0, 0]
    assert list(q[1]) == [7] + [0] * 95
    assert s[1] == F32(F32(4.875) / F32(2688.0))
    # the per-token multiplier is a rounded reciprocal: its product with amax
    # overshoots 2688 here, which is what pushes the block scale past 448
    assert F32(F32(4.875) * F32(F32(2688.0) / F32(4.875))) > F32(2688.0)
