"""ctypes binding of the C oracle (oracle/nvfp4_oracle.c).  TEST INFRASTRUCTURE ONLY.

Arrays are numpy; bf16 tensors are passed as their uint16 bit patterns.  Every function
here only marshals arguments: the arithmetic is in the C file, which cites its sources.
"""
import ctypes as C
import os

import numpy as np

from . import build_oracle

NORM = {"none": 0, "layernorm": 1, "rmsnorm": 2, "adaln": 3, "adarms": 4}
EPI = {"none": 0, "bias": 1, "residual": 2, "bias_residual": 3, "bias_gelu": 4, "geglu": 5,
       "bias_gelu_rht": 6, "geglu_rht": 7}
ROTATE, E0M3 = 1, 2  # quantizer option bits

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.orc_e2m1_decode.restype = C.c_float
        L.orc_e2m1_decode.argtypes = [C.c_uint8]
        L.orc_e2m1_encode.restype = C.c_uint8
        L.orc_e2m1_encode.argtypes = [C.c_float]
        L.orc_e4m3_decode.restype = C.c_float
        L.orc_e4m3_decode.argtypes = [C.c_uint8]
        L.orc_e4m3_encode.restype = C.c_uint8
        L.orc_e4m3_encode.argtypes = [C.c_float]
        for f in (L.orc_e2m1_encode_n, L.orc_e4m3_encode_n, L.orc_e4m3_decode_n):
            f.restype = None
            f.argtypes = [P, C.c_size_t, P]
        L.orc_sf_bytes.restype = C.c_size_t
        L.orc_sf_bytes.argtypes = [C.c_int, C.c_int]
        L.orc_sf_offset.restype = C.c_size_t
        L.orc_sf_offset.argtypes = [C.c_int, C.c_int, C.c_int]
        L.orc_quantize_block16.restype = C.c_uint8
        L.orc_quantize_block16.argtypes = [P, C.c_float, P]
        L.orc_quantize_rows.restype = None
        L.orc_quantize_rows.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_float, P, P]
        L.orc_norm_rows.restype = None
        L.orc_norm_rows.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P, P, P, P,
                                    C.c_float, P]
        L.orc_quantize_norm.restype = None
        L.orc_quantize_norm.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P, P, P,
                                        P, C.c_float, C.c_float, P, P]
        L.orc_quantize_weight.restype = C.c_float
        L.orc_quantize_weight.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, P, P]
        L.orc_block_sse.restype = C.c_double
        L.orc_block_sse.argtypes = [P, C.c_float, C.c_uint8, P]
        L.orc_quantize_block16_mse.restype = C.c_uint8
        L.orc_quantize_block16_mse.argtypes = [P, C.c_float, P]
        L.orc_quantize_weight_mse.restype = C.c_float
        L.orc_quantize_weight_mse.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, P, P]
        L.orc_dequantize.restype = None
        L.orc_dequantize.argtypes = [P, P, C.c_float, C.c_int, C.c_int, P]
        L.orc_gemm.restype = None
        L.orc_gemm.argtypes = [P, P, C.c_float, C.c_int, P, P, C.c_float, C.c_int, C.c_int,
                               C.c_int, P, P, C.c_int, P, C.c_int, P, P, C.c_float, P, P]
        L.orc_gelu_tanh.restype = C.c_double
        L.orc_gelu_tanh.argtypes = [C.c_double]
        L.orc_f32_to_bf16_array.restype = None
        L.orc_f32_to_bf16_array.argtypes = [P, C.c_size_t, P]
        L.orc_gated_residual.restype = None
        L.orc_gated_residual.argtypes = [P, P, P, C.c_int, C.c_int, P]
        L.orc_hadamard16.restype = None
        L.orc_hadamard16.argtypes = [P]
        L.orc_e0m3_decode.restype = C.c_float
        L.orc_e0m3_decode.argtypes = [C.c_uint8]
        L.orc_e0m3_encode.restype = C.c_uint8
        L.orc_e0m3_encode.argtypes = [C.c_float]
        L.orc_quantize_block16_e0m3.restype = C.c_uint8
        L.orc_quantize_block16_e0m3.argtypes = [P, C.c_float, P]
        L.orc_quantize_block16_ex.restype = C.c_uint8
        L.orc_quantize_block16_ex.argtypes = [P, C.c_float, C.c_int, P]
        L.orc_quantize_rows_ex.restype = None
        L.orc_quantize_rows_ex.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_float, C.c_int, P, P]
        L.orc_quantize_norm_ex.restype = None
        L.orc_quantize_norm_ex.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P, P, P,
                                           P, C.c_float, C.c_float, C.c_int, P, P]
        L.orc_quantize_weight_ex.restype = C.c_float
        L.orc_quantize_weight_ex.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P, P]
        L.orc_dequantize_ex.restype = None
        L.orc_dequantize_ex.argtypes = [P, P, C.c_float, C.c_int, C.c_int, C.c_int, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ---- codecs -------------------------------------------------------------------------
def e2m1_decode(codes):
    tbl = np.array([lib().orc_e2m1_decode(i) for i in range(16)], dtype=np.float32)
    return tbl[np.asarray(codes, dtype=np.uint8) & 15]


def e2m1_encode(v):
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(v), v.size, _p(out))
    return out


def e4m3_decode(c):
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_e4m3_decode_n(_p(c), c.size, _p(out))
    return out


def e4m3_encode(v):
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(v), v.size, _p(out))
    return out


# ---- layout -------------------------------------------------------------------------
def sf_bytes(rows, K):
    return int(lib().orc_sf_bytes(rows, K))


def sf_offset(row, kblk, K):
    return int(lib().orc_sf_offset(row, kblk, K))


def sf_gather(sf, rows, K):
    """Scale bytes as a dense [rows, ceil(K/16)] array (reads through the layout)."""
    nblk = (K + 15) // 16
    out = np.empty((rows, nblk), np.uint8)
    for r in range(rows):
        for b in range(nblk):
            out[r, b] = sf[sf_offset(r, b, K)]
    return out


# ---- quantizers ---------------------------------------------------------------------
def quantize_block16(y, g):
    y = _c(y, np.float32)
    assert y.size == 16
    codes = np.zeros(8, np.uint8)
    s = lib().orc_quantize_block16(_p(y), float(g), _p(codes))
    return codes, int(s)


def quantize_rows(y, g, flags=0):
    """flags: ROTATE (Hadamard-rotate each block first) | E0M3 (uniform INT4 elements)."""
    y = _c(y, np.float32)
    rows, K = y.shape
    codes = np.zeros((rows, (K + 15) // 16 * 8), np.uint8)
    sf = np.zeros(sf_bytes(rows, K), np.uint8)
    if flags:
        lib().orc_quantize_rows_ex(_p(y), rows, K, K, float(g), int(flags), _p(codes), _p(sf))
    else:
        lib().orc_quantize_rows(_p(y), rows, K, K, float(g), _p(codes), _p(sf))
    return codes, sf


def hadamard16(y):
    """The fp32 16-point Hadamard rotation of each 16-value row of y ([..., 16])."""
    y = np.array(y, dtype=np.float32, order="C")
    flat = y.reshape(-1, 16)
    for i in range(flat.shape[0]):
        lib().orc_hadamard16(flat[i].ctypes.data_as(C.c_void_p))
    return y


def e0m3_decode(codes):
    tbl = np.array([lib().orc_e0m3_decode(i) for i in range(16)], dtype=np.float32)
    return tbl[np.asarray(codes, dtype=np.uint8) & 15]


def e0m3_encode(v):
    v = np.ascontiguousarray(v, np.float32)
    return np.array([lib().orc_e0m3_encode(float(t)) for t in v.ravel()], np.uint8).reshape(v.shape)


def quantize_block16_ex(y, g, flags):
    y = _c(y, np.float32)
    assert y.size == 16
    codes = np.zeros(8, np.uint8)
    s = lib().orc_quantize_block16_ex(_p(y), float(g), int(flags), _p(codes))
    return codes, int(s)


def norm_rows(x, kind, gamma=None, beta=None, scale=None, shift=None, eps=1e-6):
    """x: uint16 (bf16 bits) or float32 [rows, K]."""
    in_fp32 = 1 if np.asarray(x).dtype == np.float32 else 0
    x = _c(x, np.float32 if in_fp32 else np.uint16)
    rows, K = x.shape
    y = np.empty((rows, K), np.float32)
    lib().orc_norm_rows(_p(x), in_fp32, rows, K, K, NORM[kind], _p(_c(gamma, np.uint16)),
                        _p(_c(beta, np.uint16)), _p(_c(scale, np.uint16)),
                        _p(_c(shift, np.uint16)), float(eps), _p(y))
    return y


def quantize_norm(x, kind, gamma=None, beta=None, scale=None, shift=None, eps=1e-6, g=1.0, flags=0):
    """flags: ROTATE | E0M3 options of the quantizer step (0: the plain NVFP4 path)."""
    in_fp32 = 1 if np.asarray(x).dtype == np.float32 else 0
    x = _c(x, np.float32 if in_fp32 else np.uint16)
    rows, K = x.shape
    codes = np.zeros((rows, (K + 15) // 16 * 8), np.uint8)
    sf = np.zeros(sf_bytes(rows, K), np.uint8)
    args = (_p(x), in_fp32, rows, K, K, NORM[kind], _p(_c(gamma, np.uint16)), _p(_c(beta, np.uint16)),
            _p(_c(scale, np.uint16)), _p(_c(shift, np.uint16)), float(eps), float(g))
    if flags:
        lib().orc_quantize_norm_ex(*args, int(flags), _p(codes), _p(sf))
    else:
        lib().orc_quantize_norm(*args, _p(codes), _p(sf))
    return codes, sf


def f32_to_bf16(v):
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().orc_f32_to_bf16_array(_p(v), v.size, _p(out))
    return out


def gated_residual(x, d, gate=None):
    """h = bf16(x + gate * d) for bf16 x, d [rows, K] and gate [K] (None: 1)."""
    x = _c(x, np.uint16)
    d = _c(d, np.uint16)
    rows, K = x.shape
    h = np.empty((rows, K), np.uint16)
    lib().orc_gated_residual(_p(x), _p(d), _p(_c(gate, np.uint16)), rows, K, _p(h))
    return h


def residual_quantize_norm(x, d, gate, kind, gamma=None, beta=None, scale=None, shift=None, eps=1e-6,
                           g=1.0):
    """The fused gated-residual front-end as its two steps: h = gated_residual(x, d, gate),
    then quantize_norm(h).  Returns (h, codes, sf)."""
    h = gated_residual(x, d, gate)
    codes, sf = quantize_norm(h, kind, gamma=gamma, beta=beta, scale=scale, shift=shift, eps=eps, g=g)
    return h, codes, sf


def quantize_weight(w, interleave_gate_up=False):
    w = _c(w, np.uint16)
    N, K = w.shape
    codes = np.zeros((N, (K + 15) // 16 * 8), np.uint8)
    sf = np.zeros(sf_bytes(N, K), np.uint8)
    g = lib().orc_quantize_weight(_p(w), N, K, K, int(bool(interleave_gate_up)), _p(codes), _p(sf))
    return codes, sf, float(np.float32(g))


def quantize_weight_mse(w, interleave_gate_up=False):
    """quantize_weight with MSE-searched block scales (the byte of least block error)."""
    w = _c(w, np.uint16)
    N, K = w.shape
    codes = np.zeros((N, (K + 15) // 16 * 8), np.uint8)
    sf = np.zeros(sf_bytes(N, K), np.uint8)
    g = lib().orc_quantize_weight_mse(_p(w), N, K, K, int(bool(interleave_gate_up)), _p(codes), _p(sf))
    return codes, sf, float(np.float32(g))


def quantize_weight_ex(w, interleave_gate_up=False, flags=0, mse=False):
    """The weight quantizer under the options (ROTATE | E0M3); mse: MSE-searched E2M1 scales."""
    w = _c(w, np.uint16)
    N, K = w.shape
    codes = np.zeros((N, (K + 15) // 16 * 8), np.uint8)
    sf = np.zeros(sf_bytes(N, K), np.uint8)
    g = lib().orc_quantize_weight_ex(_p(w), N, K, K, int(bool(interleave_gate_up)), int(flags), int(bool(mse)),
                                     _p(codes), _p(sf))
    return codes, sf, float(np.float32(g))


def block_sse(y, g, s):
    """(E(s), 8 code bytes) of one 16-value fp32 block at scale byte s."""
    y = _c(y, np.float32)
    codes = np.zeros(8, np.uint8)
    e = lib().orc_block_sse(_p(y), float(g), int(s), _p(codes))
    return float(e), codes


def quantize_block16_mse(y, g):
    y = _c(y, np.float32)
    codes = np.zeros(8, np.uint8)
    s = lib().orc_quantize_block16_mse(_p(y), float(g), _p(codes))
    return int(s), codes


def dequantize(codes, sf, g, rows, K, flags=0):
    """flags & E0M3: the codes are E0M3 (uniform INT4); a rotation is not undone."""
    codes = _c(codes, np.uint8)
    sf = _c(sf, np.uint8)
    out = np.empty((rows, K), np.float64)
    if flags:
        lib().orc_dequantize_ex(_p(codes), _p(sf), float(g), rows, K, int(flags), _p(out))
    else:
        lib().orc_dequantize(_p(codes), _p(sf), float(g), rows, K, _p(out))
    return out


def gemm(a_codes, a_sf, gA, M, w_codes, w_sf, gW, N, K, epi="none", bias=None, residual=None,
         rows=None, g_out=1.0):
    """Returns dict(v=[n_rows,N] fp64, h=[n_rows,N_out] or None, codes, sf or None)."""
    a_codes = _c(a_codes, np.uint8)
    a_sf = _c(a_sf, np.uint8)
    w_codes = _c(w_codes, np.uint8)
    w_sf = _c(w_sf, np.uint8)
    bias = _c(bias, np.uint16)
    residual = _c(residual, np.uint16)
    ldr = residual.shape[1] if residual is not None else 0
    m_idx = None if rows is None else np.ascontiguousarray(rows, np.int32)
    n_rows = M if m_idx is None else m_idx.size
    v = np.empty((n_rows, N), np.float64)
    h = codes = sf = None
    if EPI[epi] in (4, 5, 6, 7):
        n_out = N // 2 if EPI[epi] in (5, 7) else N
        h = np.empty((n_rows, n_out), np.float64)
        codes = np.zeros((M, (n_out + 15) // 16 * 8), np.uint8)
        sf = np.zeros(sf_bytes(M, n_out), np.uint8)
    lib().orc_gemm(_p(a_codes), _p(a_sf), float(gA), M, _p(w_codes), _p(w_sf), float(gW), N, K,
                   EPI[epi], _p(bias), _p(residual), ldr, _p(m_idx), n_rows, _p(v), _p(h),
                   float(g_out), _p(codes), _p(sf))
    return {"v": v, "h": h, "codes": codes, "sf": sf}


def gelu_tanh(z):
    return lib().orc_gelu_tanh(float(z))
