"""Pins for the oracle's quantizers, low-rank branch and reference GEMM (CPU).

INT4: TR-DQ section 3.1, Eq. 1-3 (uniform grid, round to nearest) in its
symmetric absmax form.  Codebook: OrbitQuant abstract (normalised rotated basis,
Lloyd-Max codes).  NVFP4: DiRotQ abstract.  Low-rank branch: DiRotQ abstract.
"""
import math

import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs

F32 = np.float32


def tree_sum(vals):
    """Recursive perfect pairwise sum in FP32 (independent restatement)."""
    if len(vals) == 1:
        return F32(vals[0])
    h = len(vals) // 2
    return F32(tree_sum(vals[:h]) + tree_sum(vals[h:]))


def test_sum_squares_order():
    rng = np.random.default_rng(0)
    y = (rng.standard_normal((3, 256)) * 10).astype(F32)
    got = orc.sum_squares(y, 64)
    for r in range(3):
        acc = None
        for blk in range(4):
            sq = [F32(v * v) for v in y[r, blk * 64:(blk + 1) * 64]]
            s = tree_sum(sq)
            acc = s if acc is None else F32(acc + s)
        assert got[r] == acc
    exact = np.sum(y.astype(np.float64) ** 2, axis=1)
    assert np.all(np.abs(got - exact) <= 4 * np.spacing(got.astype(F32)))


def test_int4_hand_cases():
    # amax 7 -> inv 1; ties at .5 go to even
    y = np.array([[7.0, 0.5, -0.5, 1.5, -2.5, 6.5, -6.5, 3.0]], dtype=F32)
    q, s = orc.quant_int4(y)
    assert list(q[0]) == [7, 0, 0, 2, -2, 6, -6, 3]
    assert s[0, 0] == F32(1.0)
    q, s = orc.quant_int4(np.zeros((1, 8), F32))
    assert s[0, 0] == 0 and not q.any()
    # per-group version: the second group is all zero
    y = np.concatenate([np.full((1, 4), 3.5, F32), np.zeros((1, 4), F32)], axis=1)
    q, s = orc.quant_int4(y, group=4)
    assert list(q[0]) == [7, 7, 7, 7, 0, 0, 0, 0] and list(s[0]) == [F32(0.5), 0.0]


def test_int4_error_bound():
    rng = np.random.default_rng(1)
    y = (rng.standard_normal((50, 128)) * rng.uniform(0.1, 10, (50, 1))).astype(F32)
    q, s = orc.quant_int4(y)
    err = np.abs(q * s[:, 0:1].astype(np.float64) - y)
    assert np.all(err <= s[:, 0:1] * 0.5 * (1 + 1e-6))
    assert np.all(np.abs(q) <= 7) and np.all(np.max(np.abs(q), axis=1) == 7)


def test_codebook_codes_count_boundaries():
    bnd = np.array([-1.0, 0.0, 1.0], dtype=F32)
    K = 4
    # row with norm 2 -> inv = sqrt(4)/2 = 1, u = y
    y = np.array([[-1.0, 0.0, 1.0, 1.4142135]], dtype=F32)
    y[0, 3] = F32(math.sqrt(4 - 2))
    codes, s = orc.quant_codebook(y, 4, bnd)
    # ties go up: u == boundary gets the upper code
    assert list(codes[0]) == [1, 2, 3, 3]
    assert s[0] == F32(np.sqrt(np.float32(np.sum(y.astype(np.float64) ** 2)))) / F32(2.0)
    codes, s = orc.quant_codebook(np.zeros((1, 4), F32), 4, bnd)
    assert list(codes[0]) == [2, 2, 2, 2] and s[0] == 0


def test_codebook_distortion_matches_lloyd_mse():
    """After RPBH every coordinate follows the sphere marginal, so the per-coordinate
    distortion of the codebook is its Lloyd-Max MSE (Gaussian-limit 16-level MSE
    is 0.009497)."""
    K, b = 3072, 128
    sign, perm = orc.make_rotation(K, b, 0)
    # isotropic input: every rotated coordinate then follows the sphere marginal
    # (heavy outlier channels stay inside their own Hadamard block and break this)
    x = np.random.default_rng(5).standard_normal((64, K)).astype(F32)
    y = orc.rotate(x, sign, perm, b)
    bf32, _ = orc.codebook_tables(K, 16)
    cent, _ = orc.lloyd_max(K, 16)
    codes, s = orc.quant_codebook(y, b, bf32)
    u = y / s[:, None]
    mse = np.mean((u - cent[codes]) ** 2)
    assert abs(mse - 0.009497) < 0.0015


def test_nvfp4_structure():
    rng = np.random.default_rng(2)
    y = (rng.standard_normal((6, 256)) * 3).astype(F32)
    y[2, 16:32] = 0
    q, sb, s = orc.quant_nvfp4(y)
    amax = np.max(np.abs(y), axis=1)
    assert np.all(s == (amax / F32(2688)).astype(F32))
    assert sb.shape == (6, 16) and sb[2, 1] == 0 and not q[2, 16:32].any()
    vals = orc.dequant_values(q, orc.NVFP4, sb)
    rec = vals * s[:, None]
    # the element with the row maximum lands on 6 * 448 (up to e4m3 rounding of its block scale)
    rel = np.abs(rec - y) / amax[:, None]
    assert np.max(rel) < 0.15
    # block maxima map near 6 in units of the block scale
    u = y * (F32(2688) / amax)[:, None]
    m16 = np.max(np.abs(u.reshape(6, 16, 16)), axis=2)
    sbv = orc.e4m3_decode(sb)
    ok = m16 > 0
    assert np.all(np.abs(m16[ok] / sbv[ok] - 6) <= 6 * 2.0 ** -3 + 1e-6)


def test_lowrank_projection_and_residual():
    w = inputs.WORKLOADS["c2"]
    x = inputs.bf16_to_f32(inputs.activations(w, M=16))
    cal = inputs.bf16_to_f32(inputs.calibration_tokens(w))
    U64, ev = orc.pca_basis(cal, 32)
    U = inputs.bf16_to_f32(inputs.bf16_bits(U64.astype(F32)))
    c = orc.project_coefficients(x, U)
    assert np.allclose(c, x.astype(np.float64) @ U.astype(np.float64), rtol=1e-5, atol=1e-3)
    cb = orc._bf16_f32(orc._bf16_bits(c))
    xr = orc.residual(x, cb, U)
    exact = x.astype(np.float64) - cb.astype(np.float64) @ U.astype(np.float64).T
    assert np.max(np.abs(xr - exact)) < 1e-4 * np.max(np.abs(exact))
    # the outlier channels live in the PCA subspace: the residual is much smaller
    assert np.max(np.abs(xr)) < 0.5 * np.max(np.abs(x))


def test_pca_basis():
    w = inputs.WORKLOADS["c2"]
    cal = inputs.bf16_to_f32(inputs.calibration_tokens(w)).astype(np.float64)
    U, ev = orc.pca_basis(cal, 32)
    assert np.allclose(U.T @ U, np.eye(32), atol=1e-12)
    S = cal.T @ cal / cal.shape[0]
    assert np.allclose(S @ U, U * ev[None, :], atol=1e-8 * ev[0])
    assert np.all(np.diff(ev) <= 0)
    idx = np.argmax(np.abs(U), axis=0)
    assert np.all(U[idx, np.arange(32)] > 0)


def brute_gemm(A, B, sa, sw, group=None):
    M, K = A.shape
    N = B.shape[0]
    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            if group:
                tot = 0.0
                for g in range(K // group):
                    part = sum(int(A[m, k]) * int(B[n, k]) for k in range(g * group, (g + 1) * group))
                    tot += part * float(sw[g][n])
                Y[m, n] = tot * float(sa[m])
            else:
                Y[m, n] = sum(float(A[m, k]) * float(B[n, k]) for k in range(K)) * float(sa[m]) * float(sw[n])
    return Y


def test_reference_gemm_int4_brute_force():
    rng = np.random.default_rng(3)
    qa = rng.integers(-7, 8, (3, 256)).astype(np.int8)
    qw = rng.integers(-7, 8, (2, 256)).astype(np.int8)
    sa = rng.uniform(0.1, 1, 3).astype(F32)
    sw = rng.uniform(0.1, 1, (2, 2)).astype(F32)
    Y = orc.reference_gemm(orc.INT4, orc.INT4, qa, sa, qw, sw)
    assert np.allclose(Y, brute_gemm(qa, qw, sa, sw, group=128), rtol=1e-14)
    # the low-rank term is added without the activation scale
    c = orc._bf16_bits(rng.standard_normal((3, 4)).astype(F32))
    L = orc._bf16_bits(rng.standard_normal((2, 4)).astype(F32))
    Y2 = orc.reference_gemm(orc.INT4, orc.INT4, qa, sa, qw, sw, c_bf16=c, L_bf16=L)
    lr = orc._bf16_f32(c).astype(np.float64) @ orc._bf16_f32(L).astype(np.float64).T
    assert np.allclose(Y2 - Y, lr, rtol=1e-12)


def test_reference_gemm_codebook_and_nvfp4_brute_force():
    rng = np.random.default_rng(4)
    cent = orc.e4m3_encode(np.linspace(-2, 2, 16).astype(F32))
    qa = rng.integers(0, 16, (2, 64)).astype(np.uint8)
    qw = rng.integers(0, 16, (3, 64)).astype(np.uint8)
    sa, sw = rng.uniform(0.5, 2, 2), rng.uniform(0.5, 2, 3)
    Y = orc.reference_gemm(orc.LM16, orc.LM16, qa, sa, qw, sw, a_cent=cent, w_cent=cent)
    v = orc.e4m3_decode(cent)
    assert np.allclose(Y, brute_gemm(v[qa], v[qw], sa, sw), rtol=1e-13)
    sba = orc.e4m3_encode(rng.uniform(0.1, 100, (2, 4)).astype(F32))
    sbw = orc.e4m3_encode(rng.uniform(0.1, 100, (3, 4)).astype(F32))
    Y = orc.reference_gemm(orc.NVFP4, orc.NVFP4, qa, sa, qw, sw, a_bs=sba, w_bs=sbw)
    A = orc.e2m1_decode(qa) * np.repeat(orc.e4m3_decode(sba), 16, axis=1)
    B = orc.e2m1_decode(qw) * np.repeat(orc.e4m3_decode(sbw), 16, axis=1)
    assert np.allclose(Y, brute_gemm(A, B, sa, sw), rtol=1e-13)


@pytest.mark.parametrize("name", ["c1", "c3", "c4", "c5"])
def test_quantized_layer_tracks_fp64_layer(name):
    """End-to-end quality of the oracle's quantized layer against x W^T (FP64):
    a transposed operand, a dropped scale or a wrong rotation blows this up."""
    w = inputs.WORKLOADS[name]
    M, N = 32, 64
    x = inputs.bf16_to_f32(inputs.activations(w, M=M))
    W = inputs.bf16_to_f32(inputs.weights(w, N=N))
    sign, perm = orc.make_rotation(w.K, w.block, 0)
    ab = wb = ac = wc = None
    if w.a_fmt in (orc.LM16,):
        ab, ac = orc.codebook_tables(w.K, 16)
    if w.w_fmt == orc.LM16:
        wb, wc = ab, ac
    if w.w_fmt == orc.LM4:
        wb, wc = orc.codebook_tables(w.K, 4)
    ra = orc.rotate_quantize(x, w.a_fmt, w.block, sign, perm, ab)
    rw = orc.rotate_quantize(W, w.w_fmt, w.block, sign, perm, wb, weight_rows=True)
    Y = orc.reference_gemm(w.a_fmt, w.w_fmt, ra["q"], ra["scale"], rw["q"], rw["scale"],
                           ra["block_scale"], rw["block_scale"], ac, wc)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    bound = {"c1": 0.25, "c3": 0.25, "c4": 0.2, "c5": 0.6}[name]
    assert rel < bound, rel
    # without the rotation the same INT4 quantizer is far worse on outlier-heavy inputs
    if name == "c1":
        qa, sa = orc.quant_int4(x)
        qw, sw = orc.quant_int4(W, group=128)
        Y0 = orc.reference_gemm(orc.INT4, orc.INT4, qa, sa[:, 0], qw, sw.T)
        rel0 = np.linalg.norm(Y0 - ref) / np.linalg.norm(ref)
        assert rel0 > 2 * rel, (rel0, rel)
