"""Pins for the oracle's DiRotQ full PCA rotation (DiRotQ abstract: activations
rotated into a calibrated PCA basis, the dominant coordinates kept in BF16, the
rest quantized, the inverse rotation folded into the weights) -- CPU only."""
import numpy as np

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs

F32 = np.float32


def _basis(K, seed=0):
    w = inputs.WORKLOADS["c2"]
    cal = inputs.bf16_to_f32(inputs.calibration_tokens(w, n=max(512, K)))[:, :K].astype(np.float64)
    S = cal.T @ cal / cal.shape[0]
    ev, V = np.linalg.eigh(S)
    V = V[:, np.argsort(ev)[::-1]]
    return inputs.bf16_to_f32(inputs.bf16_bits(V.astype(F32)))


def test_rotation_is_exact_then_rounded():
    rng = np.random.default_rng(0)
    # integer inputs: the product is exact in FP32 too
    x = rng.integers(-8, 9, (4, 64)).astype(F32)
    V = rng.integers(-4, 5, (64, 64)).astype(F32)
    assert np.array_equal(orc.rotate_pca(x, V), (x.astype(np.int64) @ V.astype(np.int64)).astype(F32))
    # BF16 inputs: equal to a float64 loop rounded once
    x = inputs.bf16_to_f32(inputs.bf16_bits(rng.standard_normal((3, 128)).astype(F32)))
    V = _basis(128)
    y = orc.rotate_pca(x, V)
    for m in range(3):
        for j in (0, 5, 127):
            acc = 0.0
            for k in range(128):
                acc += float(x[m, k]) * float(V[k, j])
            assert y[m, j] == F32(acc)


def test_split_and_folding():
    K, r = 256, 32
    V = _basis(K)
    # BF16 rounding of V leaves it orthogonal to ~2^-8
    assert np.max(np.abs(V.T.astype(np.float64) @ V - np.eye(K))) < 2e-2
    rng = np.random.default_rng(1)
    x = rng.standard_normal((8, K)).astype(F32)
    W = rng.standard_normal((16, K)).astype(F32) * F32(0.02)
    xa = orc.quantize_pca(orc.rotate_pca(x, V), r)
    wa = orc.quantize_pca(orc.rotate_pca(W, V), r, weight_rows=True)
    assert not xa["q"][:, :r].any() and not wa["q"][:, :r].any()
    Y = orc.reference_gemm(orc.INT4, orc.INT4, xa["q"], xa["scale"], wa["q"], wa["scale"], c_bf16=xa["coef"],
                           L_bf16=wa["coef"])
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.linalg.norm(Y - ref) / np.linalg.norm(ref) < 0.25
    # without the BF16 coordinates the layer loses the dominant directions
    Y0 = orc.reference_gemm(orc.INT4, orc.INT4, xa["q"], xa["scale"], wa["q"], wa["scale"])
    assert np.linalg.norm(Y0 - ref) > np.linalg.norm(Y - ref)
