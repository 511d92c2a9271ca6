"""DiRotQ's full PCA rotation on the CUDA path against the oracle (DiRotQ
abstract: activations rotated into a calibrated PCA basis, the coordinates of
the dominant directions kept in BF16, the rest quantized to 4 bits, the
inverse rotation folded into the weights).

y = x V runs on the tensor cores with FP32 accumulation in an unspecified
order, so it is held to an error bound: |y - y_exact| <= K 2^-23 sum_k
|x_k V_kn| (every product of two BF16 values is exact in FP32; each of the at
most K additions rounds by at most 2^-24 of a partial sum bounded by that
absolute sum, doubled for a truncating adder).  The split and the quantizer
that follow are bit-exact against the oracle applied to the GPU's own y; the
layer output is within 1e-3 relative Frobenius error of the oracle's FP64 sum
over the same codes."""
import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq
from tests import _harness as H

torch = pytest.importorskip("torch")

F32 = np.float32
TOL = 1e-3


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _basis_bits(w, K):
    """All K eigenvectors of the calibration tokens' second moment, dominant
    first, as BF16 bits (the oracle's PCA basis at full rank)."""
    cal = inputs.bf16_to_f32(inputs.calibration_tokens(w, n=max(512, K)))[:, :K]
    V, _ = orc.pca_basis(cal, K)
    return inputs.bf16_bits(V.astype(F32))


def _run(weight, X_bits, Vt_bits, r):
    rows, K = X_bits.shape
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty((rows, K), dtype=torch.float32, device="cuda")
    coef = torch.empty((rows, max(r, 1)), dtype=torch.int16, device="cuda")
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device="cuda")
    scale = torch.empty((K // 128, rows) if weight else (rows,), dtype=torch.float32, device="cuda")
    Xt, Vt = _dev(X_bits.view(np.int16)), _dev(Vt_bits.view(np.int16))
    fn = rq.rq_pca_quantize_weights if weight else rq.rq_pca_rotate_quantize_act
    fn(Xt, Vt, r, ws, coef if r else None, codes, scale, status)
    rc, code = rq.rq_read_status(status)
    assert rc == 0 and code == 0, hex(code)
    return {"y": ws.cpu().numpy(), "coef_t": coef, "codes_t": codes, "scale_t": scale,
            "coef": coef.cpu().numpy().view(np.uint16)[:, :r], "codes": codes.cpu().numpy(),
            "scale": scale.cpu().numpy()}


def _check_rotation(X_bits, V_bits, y_gpu):
    x = inputs.bf16_to_f32(X_bits).astype(np.float64)
    V = inputs.bf16_to_f32(V_bits).astype(np.float64)
    K = x.shape[1]
    exact = x @ V
    bound = K * 2.0 ** -23 * (np.abs(x) @ np.abs(V)) + 1e-30
    err = np.abs(y_gpu.astype(np.float64) - exact)
    assert np.all(err <= bound), float(np.max(err / bound))
    # and the oracle's rounding of the exact sum sits inside the same bound
    assert np.all(np.abs(orc.rotate_pca(inputs.bf16_to_f32(X_bits), inputs.bf16_to_f32(V_bits)) - exact) <= bound)


def _check_split(g, y, r, weight):
    o = orc.quantize_pca(y, r, weight_rows=weight)
    assert np.array_equal(g["codes"], o["codes"]), "codes differ"
    assert np.array_equal(g["scale"].view(np.uint32), o["scale"].view(np.uint32)), "scales differ"
    assert np.array_equal(g["coef"], o["coef"].reshape(g["coef"].shape)), "BF16 coordinates differ"
    return o


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N,K", [("c2", 300, 320, 1152), ("c1", 129, 256, 1152), ("c2", 64, 160, 512),
                                        ("c2", 4096, 256, 1152)])
def test_pca_layer(name, M, N, K):
    """Activations and weights through the full rotation, then the 4-bit GEMM
    with the rank-32 BF16 term; ragged M (a partial 128-row tile), K not a
    multiple of the 256-wide output tile, and the PixArt fc1 token count,
    whose product runs on 128-wide tiles (two even rounds on 148 SMs)."""
    import dataclasses
    w = dataclasses.replace(inputs.WORKLOADS[name], K=K)
    r = 32
    X = inputs.activations(w, M=M)
    W = inputs.weights(w, N=N)
    V = _basis_bits(w, K)
    Vt = np.ascontiguousarray(V.T)
    ga = _run(False, X, Vt, r)
    gw = _run(True, W, Vt, r)
    _check_rotation(X, V, ga["y"])
    _check_rotation(W, V, gw["y"])
    oa = _check_split(ga, ga["y"], r, False)
    ow = _check_split(gw, gw["y"], r, True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rq.rq_w4a4_linear(rq.INT4, rq.INT4, M, N, K, ga["codes_t"], ga["scale_t"], None, gw["codes_t"], gw["scale_t"],
                      None, None, None, ga["coef_t"], gw["coef_t"], Y, 1, status)
    assert rq.rq_read_status(status)[0] == 0
    Yref = orc.reference_gemm(orc.INT4, orc.INT4, oa["q"], oa["scale"], ow["q"], ow["scale"], c_bf16=oa["coef"],
                              L_bf16=ow["coef"])
    assert H.rel_fro(Y.cpu().numpy(), Yref) <= TOL
    # the rotation cancels inside the layer: the output tracks x W^T
    ref = inputs.bf16_to_f32(X).astype(np.float64) @ inputs.bf16_to_f32(W).astype(np.float64).T
    assert H.rel_fro(Yref, ref) < 0.25


@pytest.mark.gpu
@pytest.mark.parametrize("r", [0, 8, 200])
def test_pca_split_widths(r):
    """Other widths of the BF16 part (no GEMM: its low-rank term takes r <= 32)."""
    w = inputs.WORKLOADS["c1"]
    X = inputs.activations(w, M=70)
    V = _basis_bits(w, w.K)
    g = _run(False, X, np.ascontiguousarray(V.T), r)
    _check_rotation(X, V, g["y"])
    _check_split(g, g["y"], r, False)


@pytest.mark.gpu
def test_pca_integer_inputs_exact():
    """Small integers: every partial sum is an integer below 2^24, so any
    summation order gives the exact product (a check of the operand layouts
    that no rounding can blur)."""
    rng = np.random.default_rng(5)
    M, K = 150, 384
    x = rng.integers(-8, 9, (M, K)).astype(F32)
    V = rng.integers(-8, 9, (K, K)).astype(F32)
    g = _run(False, inputs.bf16_bits(x), inputs.bf16_bits(np.ascontiguousarray(V.T)), 16)
    assert np.array_equal(g["y"], (x.astype(np.int64) @ V.astype(np.int64)).astype(F32))


@pytest.mark.gpu
def test_pca_rejects_bad_shapes():
    w = inputs.WORKLOADS["c1"]
    X = _dev(inputs.activations(w, M=8).view(np.int16))
    Vt = torch.zeros((w.K, w.K), dtype=torch.int16, device="cuda")
    ws = torch.empty((8, w.K), dtype=torch.float32, device="cuda")
    codes = torch.empty((8, w.K // 2), dtype=torch.uint8, device="cuda")
    scale = torch.empty(8, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError):
        rq.rq_pca_rotate_quantize_act(X, Vt, w.K + 1, ws, None, codes, scale, status)
    with pytest.raises(RuntimeError):   # r > 0 without a coefficient output
        rq.rq_pca_rotate_quantize_act(X, Vt, 32, ws, None, codes, scale, status)
