"""The C-ABI library: it loads without a GPU, exports every symbol the headers in
include/ declare, its host-side preparation agrees with the oracle, and argument errors
come back before anything is launched (CPU only; no kernel runs here)."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import rq_oracle as orc
from rotated_bit_post_b200 import inputs, rq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(rq.LIB_PATH):
        from rotated_bit_post_b200 import build
        build.build()
    return rq.lib()


def declared_symbols():
    inc = os.path.join(ROOT, "include")
    src = "".join(open(os.path.join(inc, f)).read() for f in sorted(os.listdir(inc)) if f.endswith(".h"))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == {s[0] for s in rq.SIGNATURES}


@pytest.mark.parametrize("K,b,seed", [(1152, 128, 0), (3072, 128, 0), (12288, 256, 0), (1536, 128, 0), (256, 16, 9)])
def test_rotation_matches_oracle(L, K, b, seed):
    sign, perm, rot = rq.rq_make_rotation(K, b, seed)
    s2, p2 = orc.make_rotation(K, b, seed)
    assert np.array_equal(sign, s2) and np.array_equal(perm, p2)
    assert np.array_equal(rot & 0x7FFFFFFF, perm)
    assert np.array_equal((rot < 0), sign[perm] < 0)


@pytest.mark.parametrize("K,levels", [(1152, 16), (3072, 16), (1536, 16), (1536, 4), (12288, 16)])
def test_codebook_matches_oracle(L, K, levels):
    lib = rq.rq_make_codebook(K, levels)
    cent, bnd = orc.lloyd_max(K, levels)
    assert np.allclose(lib["centroids"], cent, rtol=0, atol=1e-11)
    assert np.allclose(lib["boundaries"], bnd, rtol=0, atol=1e-11)
    bf, e4 = orc.codebook_tables(K, levels)
    assert np.array_equal(lib["boundaries_f32"], bf)
    assert np.array_equal(lib["centroids_e4m3"], e4)


def test_pca_matches_oracle(L):
    w = inputs.WORKLOADS["c2"]
    cal = inputs.calibration_tokens(w)
    U, ev = rq.rq_pca_basis(cal, 32)
    Uo, evo = orc.pca_basis(inputs.bf16_to_f32(cal), 32)
    assert np.allclose(ev, evo, rtol=1e-9)
    Ul = inputs.bf16_to_f32(U).astype(np.float64)
    # equal up to BF16 rounding of the same FP64 vectors
    assert np.max(np.abs(Ul - Uo)) < 2.0 ** -8 * np.max(np.abs(Uo))
    same = np.mean(U == inputs.bf16_bits(Uo.astype(np.float32)))
    assert same > 0.999


def test_argument_errors_are_host_side(L):
    # bad block, bad K, null pointers: rejected before any device work
    code = L.rq_rotate_quantize_act(rq.INT4, None, 4, 1152, 96, None, None, None, 0, None, None, None, None, None, None)
    assert code == 2 and "block" in rq.rq_last_error()
    code = L.rq_rotate_quantize_act(rq.INT4, None, 4, 1000, 128, None, None, None, 0, None, None, None, None, None, None)
    assert code == 1
    code = L.rq_rotate_quantize_act(rq.INT4, None, 4, 1152, 128, None, None, None, 0, None, None, None, None, None, None)
    assert code == 1 and "null" in rq.rq_last_error()
    code = L.rq_rotate_quantize_act(rq.LM4, ctypes.c_void_p(16), 4, 1152, 128, ctypes.c_void_p(16), None, None, 0,
                                    None, ctypes.c_void_p(16), ctypes.c_void_p(16), None, None, None)
    assert code == 1  # 2-bit codes are for weights only
    code = L.rq_w4a4_linear(rq.INT4, rq.LM16, 4, 32, 128, *([None] * 10), 0, None, 1, None, None)
    assert code == 2
    code = L.rq_w4a4_linear(rq.INT4, rq.INT4, 4, 42, 128, *([None] * 10), 0, None, 1, None, None)
    assert code == 1 and "N=42" in rq.rq_last_error()   # INT4 weights: N % 4 == 0
    # misaligned device pointer
    p = ctypes.c_void_p(0x1008)
    code = L.rq_rotate_quantize_act(rq.INT4, p, 4, 1152, 128, p, None, None, 0, None, p, p, None, None, None)
    assert code == 3
    code = L.rq_make_rotation(1000, 128, 0, None, None, None)
    assert code == 1
    code = L.rq_make_codebook(1152, 8, None, None, None, None)
    assert code == 2


def test_k_rules_are_host_side(L):
    # K an odd multiple of 64: codebook and NVFP4 rows and GEMMs pass the shape
    # checks (and stop at the null pointers); INT4 groups need K % 128
    code = L.rq_rotate_quantize_act(rq.INT4, None, 4, 192, 64, None, None, None, 0, None, None, None, None, None, None)
    assert code == 1 and "multiple of 128" in rq.rq_last_error()
    for fmt in (rq.LM16, rq.NVFP4):
        code = L.rq_rotate_quantize_act(fmt, None, 4, 192, 64, None, None, None, 0, None, None, None, None, None, None)
        assert code == 1 and "null" in rq.rq_last_error(), rq.rq_last_error()
    code = L.rq_rotate_quantize_act(rq.LM16, None, 4, 160, 32, None, None, None, 0, None, None, None, None, None, None)
    assert code == 1 and "multiple of 64" in rq.rq_last_error()
    code = L.rq_w4a4_linear(rq.INT4, rq.INT4, 4, 32, 192, *([None] * 10), 0, None, 1, None, None)
    assert code == 1 and "multiple of 128" in rq.rq_last_error()
    for a, w in ((rq.LM16, rq.LM16), (rq.LM16, rq.LM4), (rq.NVFP4, rq.NVFP4)):
        code = L.rq_w4a4_linear(a, w, 4, 32, 192, *([None] * 10), 0, None, 1, None, None)
        assert code == 1 and "null" in rq.rq_last_error(), rq.rq_last_error()


def test_empty_batch_is_a_noop(L):
    # zero token rows (or zero weight rows) pass every argument check and return
    # RQ_OK without touching the (here fake, 16-byte aligned) device pointers
    p = ctypes.c_void_p(0x1000)
    code = L.rq_rotate_quantize_act(rq.INT4, p, 0, 1152, 128, p, None, None, 0, None, p, p, None, None, None)
    assert code == 0, rq.rq_last_error()
    code = L.rq_rotate_quantize_act(rq.NVFP4, p, 0, 1024, 256, p, None, None, 0, None, p, p, p, None, None)
    assert code == 0, rq.rq_last_error()
    code = L.rq_quantize_weights(rq.LM4, p, 0, 1536, 128, p, p, None, 0, None, p, p, None, None, None)
    assert code == 0, rq.rq_last_error()
    # the e4m3 tables are host arrays, read by the argument checks
    la = np.ascontiguousarray(rq.rq_make_codebook(1536, 16)["centroids_e4m3"], dtype=np.uint8)
    lw = np.ascontiguousarray(rq.rq_make_codebook(1536, 4)["centroids_e4m3"], dtype=np.uint8)
    hl = (la.ctypes.data_as(ctypes.c_void_p), lw.ctypes.data_as(ctypes.c_void_p))
    code = L.rq_w4a4_linear(rq.LM16, rq.LM4, 0, 256, 1536, p, p, None, p, p, None, *hl, None, None, 0, p, 0,
                            None, None)
    assert code == 0, rq.rq_last_error()
    # a negative count is still an error
    code = L.rq_w4a4_linear(rq.LM16, rq.LM4, -1, 256, 1536, p, p, None, p, p, None, *hl, None, None, 0, p, 0,
                            None, None)
    assert code == 1


def test_codebook_table_must_be_symmetric(L):
    # 16-level codes are stored sign-magnitude, so the GEMM needs the lower half
    # of its e4m3 table to mirror the upper half; checked before any launch
    p = ctypes.c_void_p(0x1000)
    cb = rq.rq_make_codebook(3072, 16)
    good = np.ascontiguousarray(cb["centroids_e4m3"], dtype=np.uint8)
    bad = good.copy()
    bad[2] ^= 0x01
    for lut, want in ((good, 0), (bad, 2)):
        code = L.rq_w4a4_linear(rq.LM16, rq.LM16, 0, 256, 3072, p, p, None, p, p, None,
                                lut.ctypes.data_as(ctypes.c_void_p), good.ctypes.data_as(ctypes.c_void_p),
                                None, None, 0, p, 0, None, None)
        assert code == want, rq.rq_last_error()
    assert "symmetric" in rq.rq_last_error()


@pytest.mark.parametrize("K,b,seed", [(8, 2, 0), (1536, 128, 1), (3072, 256, 2)])
def test_zigzag_matches_oracle(L, K, b, seed):
    rng = np.random.default_rng(seed)
    mag = rng.lognormal(0, 2, K).astype(np.float32)
    mag[::7] = mag[0]            # equal magnitudes rank by channel index on both sides
    perm, rot2 = rq.rq_make_zigzag(mag, b)
    assert np.array_equal(perm, orc.zigzag_permutation(mag, b))
    assert np.array_equal(rot2, perm)
