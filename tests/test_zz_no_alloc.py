"""The allocation-free variant of the PCA activation transform
(rq_pca_rotate_quantize_act_noalloc, built-in workspace) against the entry
point with a caller-allocated workspace, through the C ABI: two calls in a
row on different token batches, each bit-equal to the reference entry point
(codes, scales and BF16 coordinates are integers or exact FP32 bit patterns,
and both run the same kernels on the same inputs).  Collected last, and
self-contained, so that it passes alone in a fresh process as well as after
the other tests."""
import numpy as np
import pytest

from rotated_bit_post_b200 import inputs, rq

torch = pytest.importorskip("torch")


def _basis_t_bits(w):
    cal = inputs.bf16_to_f32(inputs.calibration_tokens(w, n=max(512, w.K))).astype(np.float64)
    ev, V = np.linalg.eigh(cal.T @ cal / cal.shape[0])
    V = V[:, np.argsort(ev)[::-1]]
    return inputs.bf16_bits(np.ascontiguousarray(V.T).astype(np.float32))


def _outputs(M, K, r):
    return (torch.empty((M, r), dtype=torch.int16, device="cuda"),
            torch.empty((M, K // 2), dtype=torch.uint8, device="cuda"),
            torch.empty(M, dtype=torch.float32, device="cuda"))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point():
    w = inputs.WORKLOADS["c2"]
    K, r = w.K, 32
    Vt = torch.from_numpy(_basis_t_bits(w).view(np.int16)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two batches of different lengths (the second shorter: the array keeps
    # the first call's rows beyond it)
    for row0, M in ((0, 1000), (1000, 333)):
        X = torch.from_numpy(inputs.activations(w, M=M, row0=row0).view(np.int16)).cuda()
        ws = torch.empty((M, K), dtype=torch.float32, device="cuda")
        ref = _outputs(M, K, r)
        rq.rq_pca_rotate_quantize_act(X, Vt, r, ws, *ref, status)
        got = _outputs(M, K, r)
        rq.rq_pca_rotate_quantize_act_noalloc(X, Vt, r, *got, status)
        rc, code = rq.rq_read_status(status)
        assert rc == 0 and code == 0, hex(code)
        for g, e in zip(got, ref):
            assert torch.equal(g, e)


@pytest.mark.gpu
def test_noalloc_rejects_beyond_the_limit():
    K = 1152
    M = rq.NOALLOC_MAX_ELEMS // K + 1
    X = torch.zeros((M, K), dtype=torch.int16, device="cuda")
    Vt = torch.zeros((K, K), dtype=torch.int16, device="cuda")
    c, codes, scale = _outputs(M, K, 32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(rq.RQError, match="exceeds the built-in workspace"):
        rq.rq_pca_rotate_quantize_act_noalloc(X, Vt, 32, c, codes, scale, status)
