"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Codes, scales, block scales and PCA coefficients must be
bit-exact; GEMM outputs must be within 1e-3 relative Frobenius error of the
oracle's FP64 sums over the same dequantized values (FP32 output), and the
BF16 output must be the round-to-nearest-even BF16 of the FP32 output."""
import dataclasses

import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq
from tests import _harness as H

torch = pytest.importorskip("torch")

TOL = 1e-3


def run_layer(w, M, N, row0=0, zero_rows=(), check_bf16=True):
    X = inputs.activations(w, M=M, row0=row0)
    for r in zero_rows:
        X[r] = 0
    W = inputs.weights(w, N=N)
    sign, perm, rot, cb_a, cb_w = H.tables(w)
    rot_t = torch.from_numpy(rot).cuda()
    U_t = U_f32 = None
    if w.rank:
        U64, _ = orc.pca_basis(inputs.bf16_to_f32(inputs.calibration_tokens(w)), w.rank)
        U_bits = inputs.bf16_bits(U64.astype(np.float32))
        U_t = torch.from_numpy(U_bits.view(np.int16)).cuda()
        U_f32 = inputs.bf16_to_f32(U_bits)
    ga = H.gpu_quantize(w.a_fmt, X, w.block, rot_t, None if cb_a is None else cb_a["boundaries_f32"], U_t)
    gw = H.gpu_quantize(w.w_fmt, W, w.block, rot_t, None if cb_w is None else cb_w["boundaries_f32"], U_t,
                        weight=True)
    o_sign, o_perm, ab, ac, wb, wc = H.oracle_tables(w)
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X), w.a_fmt, w.block, o_sign, o_perm, ab, U_f32)
    ow = orc.rotate_quantize(inputs.bf16_to_f32(W), w.w_fmt, w.block, o_sign, o_perm, wb, U_f32, weight_rows=True)
    H.assert_quant_equal(ga, oa, "activations")
    H.assert_quant_equal(gw, ow, "weights")
    Y = H.gpu_gemm(w, ga, gw, M, N, cb_a, cb_w, ga["coef_t"], gw["coef_t"], out_fp32=True)
    Yref = orc.reference_gemm(w.a_fmt, w.w_fmt, oa["q"], oa["scale"], ow["q"], ow["scale"], oa["block_scale"],
                              ow["block_scale"], ac, wc, oa["coef"], ow["coef"])
    Yg = Y.cpu().numpy()
    err = H.rel_fro(Yg, Yref)
    assert err <= TOL, err
    if check_bf16:
        Yb = H.gpu_gemm(w, ga, gw, M, N, cb_a, cb_w, ga["coef_t"], gw["coef_t"], out_fp32=False)
        assert torch.equal(Yb, Y.to(torch.bfloat16))
    return err


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N,row0", [
    ("c1", 256, 1152, 0),      # the full tiny PixArt-width layer
    ("c2", 200, 256, 0),       # INT4 + rank-32 branch, ragged M
    ("c3", 300, 256, 4400),    # codebook; rows straddle the image/text token boundary
    ("c4", 130, 512, 0),       # NVFP4, ragged M
    ("c5", 257, 256, 32700),   # W2A4 across the CFG branch boundary
])
def test_layer_parity(name, M, N, row0):
    run_layer(inputs.WORKLOADS[name], M, N, row0=row0)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["c1", "c3", "c4", "c5"])
def test_edge_single_row_and_zero_rows(name):
    w = inputs.WORKLOADS[name]
    run_layer(w, 1, 128 if name != "c4" else 256)
    run_layer(w, 131, 128 if name != "c4" else 256, zero_rows=(0, 77, 130))


@pytest.mark.gpu
@pytest.mark.parametrize("fmt_pair,block", [(("int4", "int4"), 128), (("lm16", "lm16"), 128),
                                            (("nvfp4", "nvfp4"), 256), (("lm16", "lm4"), 128)])
def test_edge_k_equals_block_and_narrow_n(fmt_pair, block):
    a, b = (rq.FORMATS[f] for f in fmt_pair)
    K = 256 if a == rq.NVFP4 else 128
    w = inputs.Workload("edge", 97, K, 32, block if K % block == 0 else K, a, b, 0, "pixart", "edge")
    run_layer(w, 97, 32)


@pytest.mark.gpu
def test_block_512_and_large_k():
    w = dataclasses.replace(inputs.WORKLOADS["c3"], block=512, K=4096)
    run_layer(w, 64, 128, check_bf16=False)
    w = dataclasses.replace(inputs.WORKLOADS["c4"], K=16384)
    run_layer(w, 64, 256, check_bf16=False)


@pytest.mark.gpu
@pytest.mark.parametrize("name,N", [("c3", 640), ("c5", 640), ("c5", 384), ("c4", 384), ("c1", 288), ("c2", 288)])
def test_ragged_n_after_full_tile(name, N):
    # a partial output tile after a full one: weight rows past N, their scales
    # and block scales, and (codebook) a CTA pair whose weight half is empty
    run_layer(inputs.WORKLOADS[name], 257, N)


@pytest.mark.gpu
@pytest.mark.parametrize("name,block", [("c1", 16), ("c1", 32), ("c1", 64), ("c3", 64), ("c4", 1024),
                                        ("c3", 1024), ("c5", 512)])
def test_other_block_sizes(name, block):
    # power-of-two Hadamard blocks from 16 to 1024 (TR-DQ section 3.2, Eq. 8:
    # K / 2^n blocks); blocks above 128 span several threads of the kernel
    w = dataclasses.replace(inputs.WORKLOADS[name], block=block)
    run_layer(w, 97, 256)


@pytest.mark.gpu
@pytest.mark.parametrize("name,K,block,N", [("c3", 192, 64, 256), ("c3", 64, 64, 300), ("c5", 320, 32, 640),
                                            ("c5", 64, 16, 256), ("c4", 192, 64, 256), ("c4", 320, 16, 384),
                                            ("c4", 64, 64, 128)])
def test_k_odd_multiple_of_64(name, K, block, N):
    # codebook and NVFP4 rows whose K is an odd multiple of 64: 64-wide
    # segments in the activation kernel; in the GEMM the last K step is partly
    # zero-filled by the loads and only its MMAs (and, for NVFP4, its scale
    # tiles) inside K are issued
    w = dataclasses.replace(inputs.WORKLOADS[name], K=K, block=block)
    run_layer(w, 130, N)


@pytest.mark.gpu
def test_k_multiple_of_128_where_required():
    # INT4 groups and the low-rank branch keep K % 128 == 0
    K = 192
    X = torch.zeros((4, K), dtype=torch.int16, device="cuda")
    _, _, rot = rq.rq_make_rotation(K, 64, 0)
    rot_t = torch.from_numpy(rot).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    b = rq.act_buffers(rq.INT4, 4, K)
    with pytest.raises(rq.RQError, match="multiple of 128"):
        rq.rq_rotate_quantize_act(rq.INT4, X, 64, rot_t, None, None, None, b["codes"], b["scale"], None, status)
    U = torch.zeros((K, 32), dtype=torch.int16, device="cuda")
    c = torch.empty((4, 32), dtype=torch.int16, device="cuda")
    cb = rq.rq_make_codebook(K, 16)
    b = rq.act_buffers(rq.LM16, 4, K)
    with pytest.raises(rq.RQError):
        rq.rq_rotate_quantize_act(rq.LM16, X, 64, rot_t, cb["boundaries_f32"], U, c, b["codes"], b["scale"], None,
                                  status)


@pytest.mark.gpu
@pytest.mark.parametrize("name,N", [("c3", 77), ("c5", 300), ("c5", 1), ("c4", 99), ("c1", 100), ("c2", 200),
                                    ("c3", 455)])
def test_any_n(name, N):
    # output widths that are not multiples of the tile's 32-column chunks:
    # masked element stores (N % 8 != 0: BF16 rows are not 16-byte aligned,
    # so no TMA stores), the last weight rows zero-filled by the loads; INT4
    # weights (group scales copied 16 bytes at a time) take N % 4 == 0
    run_layer(inputs.WORKLOADS[name], 130, N)


@pytest.mark.gpu
def test_int4_weights_reject_n_not_multiple_of_4():
    w = inputs.WORKLOADS["c1"]
    Y = torch.empty((8, 6), dtype=torch.float32, device="cuda")
    codes_a = torch.zeros((8, w.K // 2), dtype=torch.uint8, device="cuda")
    codes_w = torch.zeros((6, w.K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.zeros(8, dtype=torch.float32, device="cuda")
    sw = torch.zeros((w.K // 128, 6), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(rq.RQError, match="N % 4"):
        rq.rq_w4a4_linear(rq.INT4, rq.INT4, 8, 6, w.K, codes_a, sa, None, codes_w, sw, None, None, None, None, None,
                          Y, 1, status)


@pytest.mark.gpu
@pytest.mark.parametrize("name,r,K", [("c2", 8, None), ("c2", 16, None), ("c2", 24, None), ("c3", 16, None),
                                      ("c4", 16, 3072)])
def test_other_ranks(name, r, K):
    # ranks below 32 (multiples of 8): the projection pads U with zero columns
    # and the GEMM's low-rank tiles are zero-filled past r by the loads
    w = dataclasses.replace(inputs.WORKLOADS[name], rank=r)
    if K:
        w = dataclasses.replace(w, K=K)
    run_layer(w, 130, 256)
