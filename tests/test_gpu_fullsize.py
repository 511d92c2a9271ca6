"""GPU parity at the full layer sizes, in the launch configuration the benchmark
times (whole token batch and weight matrix, BF16 output, persistent tile
loop), checked on sampled outputs the oracle computes row by row.

Every row quantization is independent of the other rows, so the oracle
quantizes only the sampled activation rows and weight rows and must match the
CUDA path's codes, scales, block scales and low-rank coefficients bit for bit
there.  The sample holds one random row of every 128-token tile, one random
output column of every 128-column tile, the first and last row and column
(the ragged tails) and the rows on either side of the workload's own
boundaries (text tokens, the second guidance branch), so every output tile of
the persistent schedule is checked.  The GEMM output on the sampled grid must
be within 1e-3 relative Frobenius error of the oracle's FP64 sums, and the
BF16 output must be the round-to-nearest-even BF16 of the FP32 output."""
import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq
from tests import _harness as H

torch = pytest.importorskip("torch")

TOL = 1e-3

# rows on either side of each workload's token-range boundaries
BOUNDARY_ROWS = {"c3": (4095, 4096), "c5": (32759, 32760)}


def sample_indices(n, tile, seed, extra=()):
    """One random index in every `tile`-wide tile, plus the ends and `extra`."""
    rng = np.random.default_rng((seed, n, tile))
    idx = [t + int(rng.integers(0, min(tile, n - t))) for t in range(0, n, tile)]
    idx += [0, n - 1, *extra]
    return np.unique(np.asarray(idx, dtype=np.int64))


def unswizzled_rows(bs_t, rows_total, K, rows):
    return H.unswizzle_sf(bs_t.cpu().numpy(), rows_total, K)[rows]


@pytest.mark.gpu
@pytest.mark.slow
@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5"])
def test_full_size_sampled(name):
    w = inputs.WORKLOADS[name]
    M, N, K = w.M, w.N, w.K
    stream = torch.cuda.current_stream()
    sign, perm, rot, cb_a, cb_w = H.tables(w)
    rot_t = torch.from_numpy(rot).cuda()
    U_t = U_f32 = None
    if w.rank:
        U64, _ = orc.pca_basis(inputs.bf16_to_f32(inputs.calibration_tokens(w)), w.rank)
        U_bits = inputs.bf16_bits(U64.astype(np.float32))
        U_t = torch.from_numpy(U_bits.view(np.int16)).cuda()
        U_f32 = inputs.bf16_to_f32(U_bits)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    # ---- the CUDA path over the whole layer, as the benchmark launches it
    W = inputs.weights(w)
    wb = rq.weight_buffers(w.w_fmt, N, K, w.rank)
    rq.rq_quantize_weights(w.w_fmt, torch.from_numpy(W.view(np.int16)).cuda(), w.block, rot_t,
                           None if cb_w is None else cb_w["boundaries_f32"], U_t, wb["L"], wb["codes"], wb["scale"],
                           wb["block_scale"], status, stream)
    X = inputs.activations(w)
    ab = rq.act_buffers(w.a_fmt, M, K, w.rank)
    rq.rq_rotate_quantize_act(w.a_fmt, torch.from_numpy(X.view(np.int16)).cuda(), w.block, rot_t,
                              None if cb_a is None else cb_a["boundaries_f32"], U_t, ab["c"], ab["codes"],
                              ab["scale"], ab["block_scale"], status, stream)
    a_lut = None if cb_a is None else cb_a["centroids_e4m3"]
    w_lut = None if cb_w is None else cb_w["centroids_e4m3"]
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rq.rq_w4a4_linear(w.a_fmt, w.w_fmt, M, N, K, ab["codes"], ab["scale"], ab["block_scale"], wb["codes"],
                      wb["scale"], wb["block_scale"], a_lut, w_lut, ab["c"], wb["L"], Yb, 0, status, stream)
    Yf = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rq.rq_w4a4_linear(w.a_fmt, w.w_fmt, M, N, K, ab["codes"], ab["scale"], ab["block_scale"], wb["codes"],
                      wb["scale"], wb["block_scale"], a_lut, w_lut, ab["c"], wb["L"], Yf, 1, status, stream)
    torch.cuda.synchronize()
    rc, code = rq.rq_read_status(status)
    assert rc == 0, (rc, hex(code))

    rows = sample_indices(M, 128, 1, BOUNDARY_ROWS.get(name, ()))
    cols = sample_indices(N, 128, 2)
    rows_t = torch.from_numpy(rows).cuda()
    cols_t = torch.from_numpy(cols).cuda()

    # ---- the oracle on the sampled rows only
    o_sign, o_perm, o_ab, o_ac, o_wb, o_wc = H.oracle_tables(w)
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X[rows]), w.a_fmt, w.block, o_sign, o_perm, o_ab, U_f32)
    ow = orc.rotate_quantize(inputs.bf16_to_f32(W[cols]), w.w_fmt, w.block, o_sign, o_perm, o_wb, U_f32,
                             weight_rows=True)

    ga = {"codes": ab["codes"][rows_t].cpu().numpy(), "scale": ab["scale"][rows_t].cpu().numpy(),
          "block_scale": None if ab["block_scale"] is None else unswizzled_rows(ab["block_scale"], M, K, rows),
          "coef": None if ab["c"] is None else ab["c"][rows_t].cpu().numpy().view(np.uint16)}
    w_scale = wb["scale"][:, cols_t] if w.w_fmt == rq.INT4 else wb["scale"][cols_t]
    gw = {"codes": wb["codes"][cols_t].cpu().numpy(), "scale": w_scale.cpu().numpy(),
          "block_scale": None if wb["block_scale"] is None else unswizzled_rows(wb["block_scale"], N, K, cols),
          "coef": None if wb["L"] is None else wb["L"][cols_t].cpu().numpy().view(np.uint16)}
    H.assert_quant_equal(ga, oa, f"{name} activations")
    H.assert_quant_equal(gw, ow, f"{name} weights")

    Yref = orc.reference_gemm(w.a_fmt, w.w_fmt, oa["q"], oa["scale"], ow["q"], ow["scale"], oa["block_scale"],
                              ow["block_scale"], o_ac, o_wc, oa["coef"], ow["coef"])
    Ys = Yf[rows_t][:, cols_t]
    err = H.rel_fro(Ys.cpu().numpy(), Yref)
    assert err <= TOL, err
    # per-tile view of the same bar: no 128-row tile of the sample is off on its own
    tiles = rows // 128
    for t in np.unique(tiles):
        sel = tiles == t
        e_t = H.rel_fro(Ys.cpu().numpy()[sel], Yref[sel])
        assert e_t <= TOL, (int(t), e_t)
    assert torch.equal(Yb[rows_t][:, cols_t], Ys.to(torch.bfloat16))
