"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq


def unswizzle_sf(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Logical (rows, K/16) NVFP4 block scales from the 128x4-tile layout."""
    m = np.arange(rows)[:, None]
    kb = np.arange(K // 16)[None, :]
    off = ((m // 128) * (K // 64) + kb // 4) * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + kb % 4
    return buf[off]


def tables(w, need_a=True):
    """Rotation and codebook tables from the library (host) -- checked against
    the oracle's own in tests/test_abi.py."""
    sign, perm, rot = rq.rq_make_rotation(w.K, w.block, 0)
    cb_a = rq.rq_make_codebook(w.K, 16) if w.a_fmt == rq.LM16 else None
    cb_w = None
    if w.w_fmt == rq.LM16:
        cb_w = cb_a
    elif w.w_fmt == rq.LM4:
        cb_w = rq.rq_make_codebook(w.K, 4)
    return sign, perm, rot, cb_a, cb_w


def oracle_tables(w):
    sign, perm = orc.make_rotation(w.K, w.block, 0)
    ab = ac = wb = wc = None
    if w.a_fmt == orc.LM16:
        ab, ac = orc.codebook_tables(w.K, 16)
    if w.w_fmt == orc.LM16:
        wb, wc = ab, ac
    elif w.w_fmt == orc.LM4:
        wb, wc = orc.codebook_tables(w.K, 4)
    return sign, perm, ab, ac, wb, wc


def gpu_quantize(fmt, X_bits, block, rot_t, boundaries, U_t=None, weight=False):
    """Run K1 on BF16 bits (numpy uint16) -> dict of numpy outputs."""
    import torch
    rows, K = X_bits.shape
    X = torch.from_numpy(X_bits.view(np.int16)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = 0 if U_t is None else U_t.shape[1]
    if weight:
        b = rq.weight_buffers(fmt, rows, K, r)
        rq.rq_quantize_weights(fmt, X, block, rot_t, boundaries, U_t, b["L"], b["codes"], b["scale"],
                               b["block_scale"], status)
        coef = b["L"]
    else:
        b = rq.act_buffers(fmt, rows, K, r)
        rq.rq_rotate_quantize_act(fmt, X, block, rot_t, boundaries, U_t, b["c"], b["codes"], b["scale"],
                                  b["block_scale"], status)
        coef = b["c"]
    rc, code = rq.rq_read_status(status)
    assert rc == 0, (rc, hex(code))
    out = {"codes_t": b["codes"], "scale_t": b["scale"], "bs_t": b["block_scale"], "coef_t": coef,
           "codes": b["codes"].cpu().numpy(), "scale": b["scale"].cpu().numpy()}
    out["block_scale"] = None if b["block_scale"] is None else unswizzle_sf(b["block_scale"].cpu().numpy(), rows, K)
    out["coef"] = None if coef is None else coef.cpu().numpy().view(np.uint16)
    return out


def assert_quant_equal(g, o, label=""):
    assert g["codes"].shape == o["codes"].shape, label
    bad = np.argwhere(g["codes"] != o["codes"])
    assert bad.size == 0, f"{label}: {len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    sg = np.asarray(g["scale"], np.float32).view(np.uint32)
    so = np.asarray(o["scale"], np.float32).view(np.uint32)
    assert np.array_equal(sg, so), f"{label}: scales differ at {np.argwhere(sg != so)[:5].tolist()}"
    if o.get("block_scale") is not None:
        assert np.array_equal(g["block_scale"], o["block_scale"]), f"{label}: block scales differ"
    if o.get("coef") is not None:
        assert np.array_equal(g["coef"], o["coef"]), f"{label}: low-rank coefficients differ"


def gpu_gemm(w, ga, gw, M, N, cb_a=None, cb_w=None, c_t=None, L_t=None, out_fp32=True):
    import torch
    Y = torch.empty((M, N), dtype=torch.float32 if out_fp32 else torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rq.rq_w4a4_linear(w.a_fmt, w.w_fmt, M, N, w.K, ga["codes_t"], ga["scale_t"], ga["bs_t"], gw["codes_t"],
                      gw["scale_t"], gw["bs_t"], None if cb_a is None else cb_a["centroids_e4m3"],
                      None if cb_w is None else cb_w["centroids_e4m3"], c_t, L_t, Y, out_fp32, status)
    rc, code = rq.rq_read_status(status)
    assert rc == 0, (rc, hex(code))
    return Y


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
