"""Python binding of the C ABI in include/rq.h and include/rq_check.h (argument
marshalling only).

Every function keeps the C name.  Device buffers are torch CUDA tensors (their
data pointers are passed through); host tables are numpy arrays.  All compute
runs in the CUDA library ``librq.so``; if the library is missing or cannot be
loaded, every call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

INT4, LM16, NVFP4, LM4, INT4A, INT8 = 1, 2, 3, 4, 5, 6
NOALLOC_MAX_ELEMS = 4194304   # RQ_NOALLOC_MAX_ELEMS: the built-in workspace of the no-allocation call
FORMATS = {"int4": INT4, "lm16": LM16, "nvfp4": NVFP4, "lm4": LM4, "int4a": INT4A, "int8": INT8}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librq.so")

_lib = None

_c_i32, _c_u64, _c_p = ctypes.c_int32, ctypes.c_uint64, ctypes.c_void_p

# (name, restype, argtypes) -- mirrors include/rq.h
SIGNATURES = [
    ("rq_make_rotation", _c_i32, [_c_i32, _c_i32, _c_u64, _c_p, _c_p, _c_p]),
    ("rq_make_codebook", _c_i32, [_c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p]),
    ("rq_pca_basis", _c_i32, [_c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p]),
    ("rq_rotate_quantize_act", _c_i32,
     [_c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_quantize_weights", _c_i32,
     [_c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_w4a4_linear", _c_i32,
     [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
      _c_i32, _c_p, _c_i32, _c_p, _c_p]),
    ("rq_make_zigzag", _c_i32, [_c_p, _c_i32, _c_i32, _c_p, _c_p]),
    ("rq_rotate_quantize_act2", _c_i32,
     [_c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_quantize_weights2", _c_i32,
     [_c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_w4a4_linear2", _c_i32, [_c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p]),
    ("rq_pca_rotate_quantize_act", _c_i32, [_c_p, _c_i32, _c_i32, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_pca_quantize_weights", _c_i32, [_c_p, _c_i32, _c_i32, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_pca_rotate_quantize_act_noalloc", _c_i32, [_c_p, _c_i32, _c_i32, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_p]),
    ("rq_read_status", _c_i32, [_c_p, _c_p, _c_p]),
    ("rq_last_error", ctypes.c_char_p, []),
    # include/rq_check.h
    ("rq_convert_check", _c_i32, [_c_p, _c_i32, _c_p, _c_p, _c_p]),
    ("rq_set_wait_limit", _c_i32, [_c_u64, _c_p]),
    ("rq_set_fault_injection", _c_i32, [ctypes.c_uint32]),
]


class RQError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def lib():
    """Load librq.so (raises if it is missing: the library is the only path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run python -m rotated_bit_post_b200.build)")
        l = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _check(fn, code):
    if code != 0:
        raise RQError(fn, code, lib().rq_last_error().decode())


def _np_ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dev(t):
    """Device pointer of a torch CUDA tensor (or None)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device buffer expected (torch CUDA tensor)")
    if not t.is_contiguous():
        raise ValueError("device buffers must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------ host calls
def rq_make_rotation(K: int, block: int, seed: int = 0):
    """-> (sign int8[K], perm int32[K], rot int32[K] signed permutation)."""
    sign = np.empty(K, np.int8)
    perm = np.empty(K, np.int32)
    rot = np.empty(K, np.int32)
    _check("rq_make_rotation", lib().rq_make_rotation(K, block, seed, _np_ptr(sign), _np_ptr(perm), _np_ptr(rot)))
    return sign, perm, rot


def rq_make_codebook(K: int, levels: int):
    """-> dict(centroids f64, boundaries f64, boundaries_f32, centroids_e4m3 uint8)."""
    c = np.empty(levels, np.float64)
    b = np.empty(levels - 1, np.float64)
    bf = np.empty(levels - 1, np.float32)
    e = np.empty(levels, np.uint8)
    _check("rq_make_codebook", lib().rq_make_codebook(K, levels, _np_ptr(c), _np_ptr(b), _np_ptr(bf), _np_ptr(e)))
    return {"centroids": c, "boundaries": b, "boundaries_f32": bf, "centroids_e4m3": e}


def rq_pca_basis(calib_bf16: np.ndarray, r: int):
    """calib: uint16 BF16 bits [n, K] -> (U uint16 [K, r], eigenvalues f64 [r])."""
    calib_bf16 = np.ascontiguousarray(calib_bf16, dtype=np.uint16)
    n, K = calib_bf16.shape
    U = np.empty((K, r), np.uint16)
    ev = np.empty(r, np.float64)
    _check("rq_pca_basis", lib().rq_pca_basis(_np_ptr(calib_bf16), n, K, r, _np_ptr(U), _np_ptr(ev)))
    return U, ev


# ---------------------------------------------------------------- device calls
def rq_rotate_quantize_act(fmt, X, block, rot, boundaries, U, c_out, codes, scale, block_scale, status,
                           stream=None, r=None):
    M, K = X.shape
    bnd = None if boundaries is None else np.ascontiguousarray(boundaries, np.float32)
    rr = (U.shape[1] if U is not None else 0) if r is None else r
    _check("rq_rotate_quantize_act", lib().rq_rotate_quantize_act(
        fmt, _dev(X), M, K, block, _dev(rot), _np_ptr(bnd), _dev(U), rr, _dev(c_out), _dev(codes), _dev(scale),
        _dev(block_scale), _dev(status), _stream(stream)))


def rq_quantize_weights(fmt, W, block, rot, boundaries, U, L_out, codes, scale, block_scale, status,
                        stream=None, r=None):
    N, K = W.shape
    bnd = None if boundaries is None else np.ascontiguousarray(boundaries, np.float32)
    rr = (U.shape[1] if U is not None else 0) if r is None else r
    _check("rq_quantize_weights", lib().rq_quantize_weights(
        fmt, _dev(W), N, K, block, _dev(rot), _np_ptr(bnd), _dev(U), rr, _dev(L_out), _dev(codes), _dev(scale),
        _dev(block_scale), _dev(status), _stream(stream)))


def rq_w4a4_linear(a_fmt, w_fmt, M, N, K, a_codes, a_scale, a_bscale, w_codes, w_scale, w_bscale, a_lut, w_lut,
                   c, L, Y, out_fp32, status, stream=None):
    al = None if a_lut is None else np.ascontiguousarray(a_lut, np.uint8)
    wl = None if w_lut is None else np.ascontiguousarray(w_lut, np.uint8)
    r = 0 if c is None else c.shape[1]
    _check("rq_w4a4_linear", lib().rq_w4a4_linear(
        a_fmt, w_fmt, M, N, K, _dev(a_codes), _dev(a_scale), _dev(a_bscale), _dev(w_codes), _dev(w_scale),
        _dev(w_bscale), _np_ptr(al), _np_ptr(wl), _dev(c), _dev(L), r, _dev(Y), int(out_fp32), _dev(status),
        _stream(stream)))


def rq_make_zigzag(channel_mag: np.ndarray, block: int):
    """-> (perm int32[K], rot2 int32[K]) of TR-DQ's zigzag permutation."""
    mag = np.ascontiguousarray(channel_mag, np.float32)
    K = mag.size
    perm = np.empty(K, np.int32)
    rot2 = np.empty(K, np.int32)
    _check("rq_make_zigzag", lib().rq_make_zigzag(_np_ptr(mag), K, block, _np_ptr(perm), _np_ptr(rot2)))
    return perm, rot2


def rq_rotate_quantize_act2(fmt, X, block, rot, rot2, boundaries, codes, scale, zero_point, block_scale, status,
                            stream=None):
    M, K = X.shape
    bnd = None if boundaries is None else np.ascontiguousarray(boundaries, np.float32)
    _check("rq_rotate_quantize_act2", lib().rq_rotate_quantize_act2(
        fmt, _dev(X), M, K, block, _dev(rot), _dev(rot2), _np_ptr(bnd), _dev(codes), _dev(scale), _dev(zero_point),
        _dev(block_scale), _dev(status), _stream(stream)))


def rq_pca_rotate_quantize_act(X, Vt, r, workspace, c_out, codes, scale, status, stream=None):
    M, K = X.shape
    _check("rq_pca_rotate_quantize_act", lib().rq_pca_rotate_quantize_act(
        _dev(X), M, K, _dev(Vt), r, _dev(workspace), _dev(c_out), _dev(codes), _dev(scale), _dev(status),
        _stream(stream)))


def rq_pca_rotate_quantize_act_noalloc(X, Vt, r, c_out, codes, scale, status, stream=None):
    """rq_pca_rotate_quantize_act with the library's built-in workspace (no
    device allocation; M x K <= NOALLOC_MAX_ELEMS)."""
    M, K = X.shape
    _check("rq_pca_rotate_quantize_act_noalloc", lib().rq_pca_rotate_quantize_act_noalloc(
        _dev(X), M, K, _dev(Vt), r, _dev(c_out), _dev(codes), _dev(scale), _dev(status), _stream(stream)))


def rq_pca_quantize_weights(W, Vt, r, workspace, L_out, codes, scale, status, stream=None):
    N, K = W.shape
    _check("rq_pca_quantize_weights", lib().rq_pca_quantize_weights(
        _dev(W), N, K, _dev(Vt), r, _dev(workspace), _dev(L_out), _dev(codes), _dev(scale), _dev(status),
        _stream(stream)))


def rq_quantize_weights2(fmt, W, block, rot, rot2, boundaries, codes, scale, block_scale, zsum, status, stream=None):
    N, K = W.shape
    bnd = None if boundaries is None else np.ascontiguousarray(boundaries, np.float32)
    _check("rq_quantize_weights2", lib().rq_quantize_weights2(
        fmt, _dev(W), N, K, block, _dev(rot), _dev(rot2), _np_ptr(bnd), _dev(codes), _dev(scale),
        _dev(block_scale), _dev(zsum), _dev(status), _stream(stream)))


def rq_w4a4_linear2(M, N, K, a_codes, a_scale, a_zero_point, w_codes, w_scale, w_zsum, Y, out_fp32, status,
                    stream=None):
    _check("rq_w4a4_linear2", lib().rq_w4a4_linear2(
        M, N, K, _dev(a_codes), _dev(a_scale), _dev(a_zero_point), _dev(w_codes), _dev(w_scale), _dev(w_zsum),
        _dev(Y), int(out_fp32), _dev(status), _stream(stream)))


def rq_read_status(status, stream=None):
    code = ctypes.c_int32(0)
    rc = lib().rq_read_status(_dev(status), _stream(stream), ctypes.byref(code))
    if rc not in (0, 5):
        _check("rq_read_status", rc)
    return rc, code.value


def rq_convert_check(x, e4m3_out, e2m1_out, stream=None):
    """E4M3 bytes and E2M1 nibbles of the FP32 device tensor x, from the
    hardware conversions the activation kernel uses (include/rq_check.h)."""
    _check("rq_convert_check", lib().rq_convert_check(_dev(x), x.numel(), _dev(e4m3_out), _dev(e2m1_out),
                                                      _stream(stream)))


def rq_set_wait_limit(limit_ns: int) -> int:
    """Bound of every kernel wait for later launches (0: the 2 s default);
    returns the previous bound."""
    prev = ctypes.c_uint64(0)
    _check("rq_set_wait_limit", lib().rq_set_wait_limit(limit_ns, ctypes.byref(prev)))
    return prev.value


def rq_set_fault_injection(extra_tx_bytes: int):
    """Test hook: overstate the first operand load's byte count (0: off)."""
    _check("rq_set_fault_injection", lib().rq_set_fault_injection(extra_tx_bytes))


def rq_last_error() -> str:
    return lib().rq_last_error().decode()


# ------------------------------------------------------- buffer-size helpers
def sf_bytes(rows: int, K: int) -> int:
    """Size of an NVFP4 block-scale buffer (128-row x 64-column tiles of 512 B)."""
    return ((rows + 127) // 128) * (K // 64) * 512


def act_buffers(fmt: int, M: int, K: int, r: int = 0, device="cuda"):
    """Caller-owned output buffers for rq_rotate_quantize_act (torch, uninitialised)."""
    import torch
    out = {
        "codes": torch.empty((M, K // 2), dtype=torch.uint8, device=device),
        "scale": torch.empty(M, dtype=torch.float32, device=device),
        "block_scale": torch.zeros(sf_bytes(M, K), dtype=torch.uint8, device=device) if fmt == NVFP4 else None,
        "c": torch.empty((M, r), dtype=torch.int16, device=device) if r else None,
    }
    return out


def weight_buffers(fmt: int, N: int, K: int, r: int = 0, device="cuda"):
    import torch
    cols = K // 4 if fmt == LM4 else K // 2
    return {
        "codes": torch.empty((N, cols), dtype=torch.uint8, device=device),
        "scale": torch.empty((K // 128, N) if fmt == INT4 else (N,), dtype=torch.float32, device=device),
        "block_scale": torch.zeros(sf_bytes(N, K), dtype=torch.uint8, device=device) if fmt == NVFP4 else None,
        "L": torch.empty((N, r), dtype=torch.int16, device=device) if r else None,
    }
