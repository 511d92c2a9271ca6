"""TR-DQ on the CUDA path (TR-DQ: Time-Rotation Diffusion Quantization) against
the oracle: the double block rotation R2 P R1 with the zigzag permutation
(section 3.2, Eq. 9) on activations and weights, asymmetric per-token INT4
(section 3.1, Eq. 1-3) through the zero-point GEMM, and the timestep-indexed
selection of rotations (Eq. 10), on seeded layers of the workloads' recipes.
Codes, scales, zero points and block scales bit-exact; GEMM outputs within
1e-3 relative Frobenius error of the oracle's FP64 sums."""
import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq
from tests import _harness as H

torch = pytest.importorskip("torch")

TOL = 1e-3


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _tables_double(K, block, calib_bits, seed=0):
    """First rotation: signs only (identity permutation); second: the zigzag of
    the channel maxima after the first rotation (oracle, on calibration rows)."""
    sign, _ = orc.make_rotation(K, block, seed)
    rot1 = np.arange(K, dtype=np.int64) | np.where(sign < 0, 1 << 31, 0)
    rot1 = rot1.astype(np.uint32).view(np.int32)
    zz = orc.zigzag_from_calibration(inputs.bf16_to_f32(calib_bits), sign, block)
    perm, rot2 = rq.rq_make_zigzag(
        np.max(np.abs(orc.rotate(inputs.bf16_to_f32(calib_bits), sign, np.arange(K, dtype=np.int32), block)),
               axis=0).astype(np.float32), block)
    assert np.array_equal(perm, zz)
    return sign, rot1, zz, rot2


def _quant2(fmt, X, block, rot1, rot2, bnd=None, weight=False, zsum=False):
    rows, K = X.shape
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cols = K // 4 if fmt == rq.LM4 else K if fmt == rq.INT8 else K // 2
    codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    scale = torch.empty((K // 128, rows) if (weight and fmt == rq.INT4) else (rows,), dtype=torch.float32,
                        device="cuda")
    bs = torch.zeros(rq.sf_bytes(rows, K), dtype=torch.uint8, device="cuda") if fmt == rq.NVFP4 else None
    zp = torch.empty(rows, dtype=torch.float32, device="cuda") if fmt == rq.INT4A else None
    zs = torch.empty(rows, dtype=torch.float32, device="cuda") if zsum else None
    Xt = _dev(X.view(np.int16))
    if weight:
        rq.rq_quantize_weights2(fmt, Xt, block, rot1, rot2, bnd, codes, scale, bs, zs, status)
    else:
        rq.rq_rotate_quantize_act2(fmt, Xt, block, rot1, rot2, bnd, codes, scale, zp, bs, status)
    rc, code = rq.rq_read_status(status)
    assert rc == 0, hex(code)
    out = {"codes_t": codes, "scale_t": scale, "bs_t": bs, "zp_t": zp, "zs_t": zs,
           "codes": codes.cpu().numpy(), "scale": scale.cpu().numpy(), "coef": None}
    out["block_scale"] = None if bs is None else H.unswizzle_sf(bs.cpu().numpy(), rows, K)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("name,block,K", [("c1", 128, None), ("c3", 128, None), ("c4", 256, 3072), ("c5", 128, None),
                                          ("c1", 64, None)])
def test_double_rotation_layer(name, block, K):
    # (the FLUX down-projection shape at K = 3072: the double rotation keeps
    # an FP32 copy of each row in shared memory, so K stays at most 6144)
    import dataclasses
    w = inputs.WORKLOADS[name]
    if K:
        w = dataclasses.replace(w, K=K)
    M, N = 160, 256
    X = inputs.activations(w, M=M, row0=w.M - M if name == "c5" else 0)
    W = inputs.weights(w, N=N)
    sign, rot1, zz, rot2 = _tables_double(w.K, block, inputs.calibration_tokens(w))
    r1, r2 = _dev(rot1), _dev(rot2)
    cb_a = orc.codebook_tables(w.K, 16) if w.a_fmt == rq.LM16 else (None, None)
    cb_w = cb_a if w.w_fmt == rq.LM16 else (orc.codebook_tables(w.K, 4) if w.w_fmt == rq.LM4 else (None, None))
    ga = _quant2(w.a_fmt, X, block, r1, r2, cb_a[0])
    gw = _quant2(w.w_fmt, W, block, r1, r2, cb_w[0], weight=True)
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X), w.a_fmt, block, sign, None, cb_a[0], zz_perm=zz)
    ow = orc.rotate_quantize(inputs.bf16_to_f32(W), w.w_fmt, block, sign, None, cb_w[0], weight_rows=True,
                             zz_perm=zz)
    H.assert_quant_equal(ga, oa, "activations")
    H.assert_quant_equal(gw, ow, "weights")
    Y = H.gpu_gemm(w, ga, gw, M, N, None if cb_a[1] is None else {"centroids_e4m3": cb_a[1]},
                   None if cb_w[1] is None else {"centroids_e4m3": cb_w[1]})
    Yref = orc.reference_gemm(w.a_fmt, w.w_fmt, oa["q"], oa["scale"], ow["q"], ow["scale"], oa["block_scale"],
                              ow["block_scale"], cb_a[1], cb_w[1])
    assert H.rel_fro(Y.cpu().numpy(), Yref) <= TOL
    # the double rotation cancels inside the layer like the single one: the
    # quantized layer tracks x W^T as closely (TR-DQ Eq. 9)
    # (the same bounds as the oracle's single-rotation check; W2A4 is coarser)
    ref = inputs.bf16_to_f32(X).astype(np.float64) @ inputs.bf16_to_f32(W).astype(np.float64).T
    assert H.rel_fro(Yref, ref) < {"c1": 0.25, "c3": 0.25, "c4": 0.2, "c5": 0.6}[name]


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N,double", [("c1", 256, 1152, False), ("c2", 300, 512, False),
                                             ("c1", 200, 384, True)])
def test_asymmetric_int4_layer(name, M, N, double):
    w = inputs.WORKLOADS[name]
    X = inputs.activations(w, M=M)
    W = inputs.weights(w, N=N)
    if double:
        sign, rot1, zz, rot2 = _tables_double(w.K, w.block, inputs.calibration_tokens(w))
        r2 = _dev(rot2)
        o_sign, o_perm = sign, None
    else:
        o_sign, o_perm = orc.make_rotation(w.K, w.block, 0)
        _, _, rot1 = rq.rq_make_rotation(w.K, w.block, 0)
        zz, r2 = None, None
    r1 = _dev(rot1)
    ga = _quant2(rq.INT4A, X, w.block, r1, r2)
    gw = _quant2(rq.INT4, W, w.block, r1, r2, weight=True, zsum=True)
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X), orc.INT4A, w.block, o_sign, o_perm, zz_perm=zz)
    ow = orc.rotate_quantize(inputs.bf16_to_f32(W), orc.INT4, w.block, o_sign, o_perm, weight_rows=True, zz_perm=zz)
    H.assert_quant_equal(ga, oa, "activations")
    H.assert_quant_equal(gw, ow, "weights")
    assert np.array_equal(ga["zp_t"].cpu().numpy().view(np.uint32), oa["zero_point"].view(np.uint32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for out_fp32 in (1, 0):
        Y = torch.empty((M, N), dtype=torch.float32 if out_fp32 else torch.bfloat16, device="cuda")
        rq.rq_w4a4_linear2(M, N, w.K, ga["codes_t"], ga["scale_t"], ga["zp_t"], gw["codes_t"], gw["scale_t"],
                           gw["zs_t"], Y, out_fp32, status)
        assert rq.rq_read_status(status)[0] == 0
        if out_fp32:
            Yf = Y
            Yref = orc.reference_gemm(orc.INT4A, orc.INT4, oa["q"], oa["scale"], ow["q"], ow["scale"],
                                      a_zp=oa["zero_point"])
            assert H.rel_fro(Y.cpu().numpy(), Yref) <= TOL
        else:
            assert torch.equal(Y, Yf.to(torch.bfloat16))


@pytest.mark.gpu
def test_timestep_rotation_selection():
    # Eq. 10: each timestep t has its own rotation (and weights folded with
    # it); selecting t selects that table.  Two timesteps' tables side by side
    # in one device buffer; the call for step t gets the slice of step t.
    w = inputs.WORKLOADS["c1"]
    M, N = 128, 256
    X = inputs.activations(w, M=M)
    W = inputs.weights(w, N=N)
    rots = []
    for t in range(2):
        _, _, rot = rq.rq_make_rotation(w.K, w.block, 100 + t)
        rots.append(rot)
    table = _dev(np.concatenate(rots))
    outs = []
    for t in range(2):
        rot_t = table[t * w.K:(t + 1) * w.K]
        ga = _quant2(rq.INT4, X, w.block, rot_t, None)
        gw = _quant2(rq.INT4, W, w.block, rot_t, None, weight=True)
        sign, perm = orc.make_rotation(w.K, w.block, 100 + t)
        oa = orc.rotate_quantize(inputs.bf16_to_f32(X), orc.INT4, w.block, sign, perm)
        H.assert_quant_equal(ga, oa, f"step {t}")
        outs.append(H.gpu_gemm(w, ga, gw, M, N).cpu().numpy())
    ref = inputs.bf16_to_f32(X).astype(np.float64) @ inputs.bf16_to_f32(W).astype(np.float64).T
    assert not np.array_equal(outs[0], outs[1])
    assert H.rel_fro(outs[0], ref) < 0.3 and H.rel_fro(outs[1], ref) < 0.3


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N", [("c1", 256, 1152), ("c2", 300, 640), ("c3", 130, 256)])
def test_w4a8_layer(name, M, N):
    # TR-DQ's W4A8 setting (Tables 1-5): 8-bit per-token activations against
    # INT4 weights with one scale per 128 rotated coordinates
    w = inputs.WORKLOADS[name]
    X = inputs.activations(w, M=M)
    W = inputs.weights(w, N=N)
    o_sign, o_perm = orc.make_rotation(w.K, w.block, 0)
    _, _, rot = rq.rq_make_rotation(w.K, w.block, 0)
    r1 = _dev(rot)
    ga = _quant2(rq.INT8, X, w.block, r1, None)
    gw = _quant2(rq.INT4, W, w.block, r1, None, weight=True)
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X), orc.INT8, w.block, o_sign, o_perm)
    ow = orc.rotate_quantize(inputs.bf16_to_f32(W), orc.INT4, w.block, o_sign, o_perm, weight_rows=True)
    H.assert_quant_equal(ga, oa, "activations")
    H.assert_quant_equal(gw, ow, "weights")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for Y, f in ((Yf, 1), (Yb, 0)):
        rq.rq_w4a4_linear(rq.INT8, rq.INT4, M, N, w.K, ga["codes_t"], ga["scale_t"], None, gw["codes_t"],
                          gw["scale_t"], None, None, None, None, None, Y, f, status)
        assert rq.rq_read_status(status)[0] == 0
    Yref = orc.reference_gemm(orc.INT8, orc.INT4, oa["q"], oa["scale"], ow["q"], ow["scale"])
    assert H.rel_fro(Yf.cpu().numpy(), Yref) <= TOL
    assert torch.equal(Yb, Yf.to(torch.bfloat16))
    # 8-bit activations track x W^T more closely than 4-bit ones
    ref = inputs.bf16_to_f32(X).astype(np.float64) @ inputs.bf16_to_f32(W).astype(np.float64).T
    o4 = orc.rotate_quantize(inputs.bf16_to_f32(X), orc.INT4, w.block, o_sign, o_perm)
    Y4 = orc.reference_gemm(orc.INT4, orc.INT4, o4["q"], o4["scale"], ow["q"], ow["scale"])
    assert H.rel_fro(Yref, ref) < H.rel_fro(Y4, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N", [("c1", 256, 1152), ("c2", 300, 640), ("c3", 130, 288)])
def test_w8a8_layer(name, M, N):
    # TR-DQ's W8A8 setting (Tables 1-5; section 3.1: per-token activations,
    # per-channel weights): both operands 8-bit, one dense kind::i8 GEMM
    w = inputs.WORKLOADS[name]
    X = inputs.activations(w, M=M)
    W = inputs.weights(w, N=N)
    o_sign, o_perm = orc.make_rotation(w.K, w.block, 0)
    _, _, rot = rq.rq_make_rotation(w.K, w.block, 0)
    r1 = _dev(rot)
    ga = _quant2(rq.INT8, X, w.block, r1, None)
    gw = _quant2(rq.INT8, W, w.block, r1, None, weight=True)
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X), orc.INT8, w.block, o_sign, o_perm)
    ow = orc.rotate_quantize(inputs.bf16_to_f32(W), orc.INT8, w.block, o_sign, o_perm, weight_rows=True)
    H.assert_quant_equal(ga, oa, "activations")
    H.assert_quant_equal(gw, ow, "weights")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for Y, f in ((Yf, 1), (Yb, 0)):
        rq.rq_w4a4_linear(rq.INT8, rq.INT8, M, N, w.K, ga["codes_t"], ga["scale_t"], None, gw["codes_t"],
                          gw["scale_t"], None, None, None, None, None, Y, f, status)
        assert rq.rq_read_status(status)[0] == 0
    Yref = orc.reference_gemm(orc.INT8, orc.INT8, oa["q"], oa["scale"], ow["q"], ow["scale"])
    assert H.rel_fro(Yf.cpu().numpy(), Yref) <= TOL
    assert torch.equal(Yb, Yf.to(torch.bfloat16))
    # 8-bit weights track x W^T more closely than 4-bit ones
    ref = inputs.bf16_to_f32(X).astype(np.float64) @ inputs.bf16_to_f32(W).astype(np.float64).T
    o4 = orc.rotate_quantize(inputs.bf16_to_f32(W), orc.INT4, w.block, o_sign, o_perm, weight_rows=True)
    Y4 = orc.reference_gemm(orc.INT8, orc.INT4, oa["q"], oa["scale"], o4["q"], o4["scale"])
    assert H.rel_fro(Yref, ref) < H.rel_fro(Y4, ref)
