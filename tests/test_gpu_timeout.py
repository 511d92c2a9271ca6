"""Failure detection on the GPU without a fault: a wait that runs out.

The library's test hook makes the first operand load of every CTA announce 16
more bytes than its copies bring (every copy still lands), so the kernels'
bounded waits on that barrier run out after the wait limit, here 5 ms.  The
call must then report RQ_ERR_TIMEOUT through rq_read_status with the code of
the wait that gave up, and the next normal call on the same stream must give
the same result as a call made before the injection (bit for bit)."""
import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq
from tests import _harness as H

torch = pytest.importorskip("torch")

RQ_ERR_TIMEOUT = 5
TIMEOUT_CODES = {0x101, 0x102, 0x103, 0x104, 0x105}


class injected:
    def __enter__(self):
        rq.rq_set_wait_limit(5_000_000)
        rq.rq_set_fault_injection(16)

    def __exit__(self, *exc):
        rq.rq_set_fault_injection(0)
        rq.rq_set_wait_limit(0)


def _layer(name, M, N):
    w = inputs.WORKLOADS[name]
    X = inputs.activations(w, M=M)
    W = inputs.weights(w, N=N)
    sign, perm, rot, cb_a, cb_w = H.tables(w)
    rot_t = torch.from_numpy(rot).cuda()
    a_bnd = None if cb_a is None else cb_a["boundaries_f32"]
    w_bnd = None if cb_w is None else cb_w["boundaries_f32"]
    ga = H.gpu_quantize(w.a_fmt, X, w.block, rot_t, a_bnd)
    gw = H.gpu_quantize(w.w_fmt, W, w.block, rot_t, w_bnd, weight=True)
    return w, X, rot_t, a_bnd, ga, gw, cb_a, cb_w


def _gemm(w, ga, gw, M, N, cb_a, cb_w, status):
    Y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    rq.rq_w4a4_linear(w.a_fmt, w.w_fmt, M, N, w.K, ga["codes_t"], ga["scale_t"], ga["bs_t"], gw["codes_t"],
                      gw["scale_t"], gw["bs_t"], None if cb_a is None else cb_a["centroids_e4m3"],
                      None if cb_w is None else cb_w["centroids_e4m3"], None, None, Y, 1, status)
    return Y


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["c1", "c3", "c4", "c5"])
def test_gemm_wait_runs_out_then_recovers(name):
    M, N = 300, 512
    w, X, rot_t, a_bnd, ga, gw, cb_a, cb_w = _layer(name, M, N)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y0 = _gemm(w, ga, gw, M, N, cb_a, cb_w, status)
    assert rq.rq_read_status(status)[0] == 0
    with injected():
        _gemm(w, ga, gw, M, N, cb_a, cb_w, status)
        rc, code = rq.rq_read_status(status)
    assert rc == RQ_ERR_TIMEOUT and code in TIMEOUT_CODES, (rc, hex(code))
    status.zero_()
    Y1 = _gemm(w, ga, gw, M, N, cb_a, cb_w, status)
    assert rq.rq_read_status(status)[0] == 0
    assert torch.equal(Y0, Y1)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["c1", "c4"])
def test_activation_wait_runs_out_then_recovers(name):
    w = inputs.WORKLOADS[name]
    X = inputs.activations(w, M=200)
    sign, perm, rot, cb_a, cb_w = H.tables(w)
    rot_t = torch.from_numpy(rot).cuda()
    Xt = torch.from_numpy(X.view(np.int16)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    b = rq.act_buffers(w.a_fmt, 200, w.K)
    with injected():
        rq.rq_rotate_quantize_act(w.a_fmt, Xt, w.block, rot_t, None, None, None, b["codes"], b["scale"],
                                  b["block_scale"], status)
        rc, code = rq.rq_read_status(status)
    assert rc == RQ_ERR_TIMEOUT and code == 0x105, (rc, hex(code))
    status.zero_()
    g = H.gpu_quantize(w.a_fmt, X, w.block, rot_t, None)
    o = orc.rotate_quantize(inputs.bf16_to_f32(X), w.a_fmt, w.block, sign, perm, None)
    H.assert_quant_equal(g, o, name)
