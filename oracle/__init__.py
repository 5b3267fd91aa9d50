"""ctypes front-end of the libbsq CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``.  The library path never imports
it, and it imports nothing from the library.

Every array is a numpy array; BF16 tensors are ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Plain IEEE float: no contraction into FMA, no fast-math.
CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
          "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (seconds)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_u8p = ctypes.POINTER(ctypes.c_uint8)
_i8p = ctypes.POINTER(ctypes.c_int8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def _declare(L):
    L.or_e2m1_value.restype = ctypes.c_double
    L.or_e2m1_value.argtypes = [ctypes.c_uint8]
    L.or_e4m3_value.restype = ctypes.c_double
    L.or_e4m3_value.argtypes = [ctypes.c_uint8]
    L.or_e2m1_encode.restype = ctypes.c_uint8
    L.or_e2m1_encode.argtypes = [ctypes.c_float]
    L.or_e4m3_encode.restype = ctypes.c_uint8
    L.or_e4m3_encode.argtypes = [ctypes.c_float]
    L.or_bf16_encode.restype = ctypes.c_uint16
    L.or_bf16_encode.argtypes = [ctypes.c_double]
    L.or_bf16_value.restype = ctypes.c_float
    L.or_bf16_value.argtypes = [ctypes.c_uint16]
    L.or_num_threads.restype = ctypes.c_int
    L.or_amax_bf16.restype = ctypes.c_float
    L.or_amax_bf16.argtypes = [_u16p, _i64]
    L.or_quant_nvfp4.argtypes = [_u16p, _i64, _i64, ctypes.c_float, _u8p, _u8p]
    L.or_quant_rowwise_fp8.argtypes = [_u16p, _i64, _i64, _u8p, _f32p]
    L.or_quant_blockfp8.argtypes = [_u16p, _i64, _i64, _u8p, _f32p]
    L.or_requant_w_nvfp4_int8.argtypes = [_u8p, _u8p, ctypes.c_float, _i64, _i64, _i8p, _f32p]
    L.or_quant_act_int8_per32.argtypes = [_u16p, _i64, _i64, _i8p, _f32p]
    L.or_requant_blockfp8_to_rowwise.argtypes = [_u8p, _f32p, _i64, _i64, _u8p, _f32p]
    prod_tail = [_i64, _i64, _i64, _i64p, _i64, _u16p, _f64p, _f64p]
    L.or_w4a4_gemm.argtypes = [_u8p, _u8p, _u8p, _u8p, ctypes.c_float, ctypes.c_float] + prod_tail
    L.or_fp8_gemv_rowscale.argtypes = [_u16p, _u8p, _f32p] + prod_tail
    L.or_fp8_gemv_blockscaled.argtypes = [_u16p, _u8p, _f32p] + prod_tail
    L.or_int8_blockscaled_gemm.argtypes = [_i8p, _i8p, _f32p, _f32p] + prod_tail
    L.or_fp8_gemm_rowscale.argtypes = [_u8p, _f32p, _u8p, _f32p] + prod_tail


def _p(a, ptype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ptype)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- codecs -----------------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().or_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().or_e4m3_value(code)


def e2m1_encode(x: float) -> int:
    return lib().or_e2m1_encode(x)


def e4m3_encode(x: float) -> int:
    return lib().or_e4m3_encode(x)


def bf16_encode(x: float) -> int:
    return lib().or_bf16_encode(x)


def bf16_value(b: int) -> float:
    return lib().or_bf16_value(b)


def num_threads() -> int:
    return lib().or_num_threads()


# ---- quantisers -------------------------------------------------------------

def quant_nvfp4(x_bf16: np.ndarray, scale2: float):
    x = _c(x_bf16, np.uint16)
    rows, k = x.shape
    packed = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros((rows, k // 16), np.uint8)
    lib().or_quant_nvfp4(_p(x, _u16p), rows, k, scale2, _p(packed, _u8p), _p(sf, _u8p))
    return packed, sf


def quant_rowwise_fp8(x_bf16: np.ndarray):
    x = _c(x_bf16, np.uint16)
    rows, k = x.shape
    q = np.zeros((rows, k), np.uint8)
    s = np.zeros((rows,), np.float32)
    lib().or_quant_rowwise_fp8(_p(x, _u16p), rows, k, _p(q, _u8p), _p(s, _f32p))
    return q, s


def quant_blockfp8(x_bf16: np.ndarray):
    x = _c(x_bf16, np.uint16)
    n, k = x.shape
    q = np.zeros((n, k), np.uint8)
    s = np.zeros((n // 128, k // 128), np.float32)
    lib().or_quant_blockfp8(_p(x, _u16p), n, k, _p(q, _u8p), _p(s, _f32p))
    return q, s


def requant_w_nvfp4_int8(packed: np.ndarray, sf: np.ndarray, scale2: float):
    packed = _c(packed, np.uint8)
    sf = _c(sf, np.uint8)
    n, k = packed.shape[0], packed.shape[1] * 2
    q = np.zeros((n, k), np.int8)
    s = np.zeros((n, k // 32), np.float32)
    lib().or_requant_w_nvfp4_int8(_p(packed, _u8p), _p(sf, _u8p), scale2, n, k,
                                  _p(q, _i8p), _p(s, _f32p))
    return q, s


def quant_act_int8_per32(x_bf16: np.ndarray):
    x = _c(x_bf16, np.uint16)
    m, k = x.shape
    q = np.zeros((m, k), np.int8)
    s = np.zeros((m, k // 32), np.float32)
    lib().or_quant_act_int8_per32(_p(x, _u16p), m, k, _p(q, _i8p), _p(s, _f32p))
    return q, s


def requant_blockfp8_to_rowwise(w: np.ndarray, bscale: np.ndarray):
    w = _c(w, np.uint8)
    bscale = _c(bscale, np.float32)
    n, k = w.shape
    q = np.zeros((n, k), np.uint8)
    s = np.zeros((n,), np.float32)
    lib().or_requant_blockfp8_to_rowwise(_p(w, _u8p), _p(bscale, _f32p), n, k,
                                         _p(q, _u8p), _p(s, _f32p))
    return q, s


def amax_bf16(x_bf16: np.ndarray) -> float:
    x = _c(x_bf16, np.uint16)
    return lib().or_amax_bf16(_p(x, _u16p), x.size)


# ---- products ---------------------------------------------------------------

def _prod_out(rows, m, n):
    if rows is None:
        r = None
        nr = m
    else:
        r = _c(rows, np.int64)
        nr = r.size
    return r, nr, np.zeros((nr, n), np.uint16), np.zeros((nr, n)), np.zeros((nr, n))


def w4a4_gemm(a_packed, a_sf, w_packed, w_sf, scale_a2, scale_b2, rows=None):
    """Returns (out_bf16 [nr,n] uint16, exact [nr,n] f64, abssum [nr,n] f64)."""
    a_packed, a_sf = _c(a_packed, np.uint8), _c(a_sf, np.uint8)
    w_packed, w_sf = _c(w_packed, np.uint8), _c(w_sf, np.uint8)
    m, k = a_packed.shape[0], a_packed.shape[1] * 2
    n = w_packed.shape[0]
    r, nr, ob, oe, oa = _prod_out(rows, m, n)
    lib().or_w4a4_gemm(_p(a_packed, _u8p), _p(a_sf, _u8p), _p(w_packed, _u8p), _p(w_sf, _u8p),
                       scale_a2, scale_b2, m, n, k, _p(r, _i64p), nr,
                       _p(ob, _u16p), _p(oe, _f64p), _p(oa, _f64p))
    return ob, oe, oa


def fp8_gemv_rowscale(inp_bf16, w, row_scale, rows=None):
    inp, w = _c(inp_bf16, np.uint16), _c(w, np.uint8)
    row_scale = _c(row_scale, np.float32)
    m, k = inp.shape
    n = w.shape[0]
    r, nr, ob, oe, oa = _prod_out(rows, m, n)
    lib().or_fp8_gemv_rowscale(_p(inp, _u16p), _p(w, _u8p), _p(row_scale, _f32p),
                               m, n, k, _p(r, _i64p), nr,
                               _p(ob, _u16p), _p(oe, _f64p), _p(oa, _f64p))
    return ob, oe, oa


def fp8_gemv_blockscaled(inp_bf16, w, block_scale, rows=None):
    """Block-scaled FP8 GEMV: block_scale is the FP32 grid [N/128, K/128]."""
    inp, w = _c(inp_bf16, np.uint16), _c(w, np.uint8)
    block_scale = _c(block_scale, np.float32)
    m, k = inp.shape
    n = w.shape[0]
    assert n % 128 == 0 and k % 128 == 0 and block_scale.shape == (n // 128, k // 128)
    r, nr, ob, oe, oa = _prod_out(rows, m, n)
    lib().or_fp8_gemv_blockscaled(_p(inp, _u16p), _p(w, _u8p), _p(block_scale, _f32p),
                                  m, n, k, _p(r, _i64p), nr,
                                  _p(ob, _u16p), _p(oe, _f64p), _p(oa, _f64p))
    return ob, oe, oa


def int8_blockscaled_gemm(a, w, a_scale, w_scale, rows=None):
    a, w = _c(a, np.int8), _c(w, np.int8)
    a_scale, w_scale = _c(a_scale, np.float32), _c(w_scale, np.float32)
    m, k = a.shape
    n = w.shape[0]
    r, nr, ob, oe, oa = _prod_out(rows, m, n)
    lib().or_int8_blockscaled_gemm(_p(a, _i8p), _p(w, _i8p), _p(a_scale, _f32p), _p(w_scale, _f32p),
                                   m, n, k, _p(r, _i64p), nr,
                                   _p(ob, _u16p), _p(oe, _f64p), _p(oa, _f64p))
    return ob, oe, oa


def fp8_gemm_rowscale(a, a_scale, w, w_scale, rows=None):
    a, w = _c(a, np.uint8), _c(w, np.uint8)
    a_scale, w_scale = _c(a_scale, np.float32), _c(w_scale, np.float32)
    m, k = a.shape
    n = w.shape[0]
    r, nr, ob, oe, oa = _prod_out(rows, m, n)
    lib().or_fp8_gemm_rowscale(_p(a, _u8p), _p(a_scale, _f32p), _p(w, _u8p), _p(w_scale, _f32p),
                               m, n, k, _p(r, _i64p), nr,
                               _p(ob, _u16p), _p(oe, _f64p), _p(oa, _f64p))
    return ob, oe, oa


def tolerance(oracle_bf16: np.ndarray, abssum: np.ndarray) -> np.ndarray:
    """|gpu - oracle| bound: 1e-2 * |oracle| + 1e-3 * sum|a*w|."""
    o = bf16_to_f32(oracle_bf16).astype(np.float64)
    return 1e-2 * np.abs(o) + 1e-3 * abssum


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)
