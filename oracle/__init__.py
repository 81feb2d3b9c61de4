"""CPU oracle for the NVFP4 W4A4 linear -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``nvfp4_block_scaled_17_b200``) never imports it and shares no code with it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp32 operations in the
order the readings fix, fp64 for the GEMM).  This module only compiles it and
marshals numpy arrays.  bf16 tensors travel as ``uint16`` bit patterns.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against things fixed outside the oracle (library casts, closed forms, brute
force, the pages' printed figures).  None is left "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnvfp4_oracle.so")
_lib = None

u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle shared library next to its source (gcc, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".{os.getpid()}.tmp"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
           "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.ora_bf16_to_f32.restype = ctypes.c_float
        L.ora_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.ora_f32_to_bf16.restype = ctypes.c_uint16
        L.ora_f32_to_bf16.argtypes = [ctypes.c_float]
        L.ora_e2m1_decode.restype = ctypes.c_double
        L.ora_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.ora_e2m1_encode.restype = ctypes.c_uint8
        L.ora_e2m1_encode.argtypes = [ctypes.c_float]
        L.ora_e4m3_decode.restype = ctypes.c_double
        L.ora_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.ora_e4m3_encode.restype = ctypes.c_uint8
        L.ora_e4m3_encode.argtypes = [ctypes.c_float]
        L.ora_amax_bf16.restype = ctypes.c_float
        L.ora_amax_bf16.argtypes = [u16p, ctypes.c_int64]
        L.ora_global_scale.restype = ctypes.c_float
        L.ora_global_scale.argtypes = [ctypes.c_float]
        L.ora_alpha.restype = ctypes.c_float
        L.ora_alpha.argtypes = [ctypes.c_float, ctypes.c_float]
        L.ora_quantize_rows.restype = None
        L.ora_quantize_rows.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float,
                                        u8p, u8p]
        for name in ("ora_scale_rows_padded", "ora_scale_cols_padded"):
            getattr(L, name).restype = ctypes.c_int64
            getattr(L, name).argtypes = [ctypes.c_int64]
        L.ora_scale_bytes.restype = ctypes.c_int64
        L.ora_scale_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        L.ora_scale_offset.restype = ctypes.c_int64
        L.ora_scale_offset.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.ora_scale_swizzle.restype = None
        L.ora_scale_swizzle.argtypes = [u8p, ctypes.c_int64, ctypes.c_int64, u8p]
        L.ora_scale_unswizzle.restype = None
        L.ora_scale_unswizzle.argtypes = [u8p, ctypes.c_int64, ctypes.c_int64, u8p]
        L.ora_hadamard_scale.restype = ctypes.c_float
        L.ora_hadamard_scale.argtypes = [ctypes.c_int]
        L.ora_hadamard_rotate.restype = None
        L.ora_hadamard_rotate.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, u16p]
        L.ora_dequantize.restype = None
        L.ora_dequantize.argtypes = [u8p, u8p, ctypes.c_int64, ctypes.c_int64, f64p]
        i8p = np.ctypeslib.ndpointer(dtype=np.int8, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
        L.ora_int8_quantize_rows.restype = None
        L.ora_int8_quantize_rows.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, i8p, f32p]
        L.ora_int8_gemm_f64.restype = None
        L.ora_int8_gemm_f64.argtypes = [i8p, f32p, i8p, f32p, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, f64p]
        L.ora_dequantize_bf16.restype = None
        L.ora_dequantize_bf16.argtypes = [u8p, u8p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float,
                                          u16p]
        L.ora_gemm_f64.restype = None
        L.ora_gemm_f64.argtypes = [u8p, u8p, u8p, u8p, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int64, f64p]
        for name in ("ora_e2m1_encode_array", "ora_e4m3_encode_array"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [f32p, ctypes.c_int64, u8p]
        L.ora_f32_to_bf16_array.restype = None
        L.ora_f32_to_bf16_array.argtypes = [f32p, ctypes.c_int64, u16p]
        L.ora_quantize.restype = ctypes.c_float
        L.ora_quantize.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float,
                                   u8p, u8p, u8p]
    return _lib


# --------------------------------------------------------------------------
# scalar formats
# --------------------------------------------------------------------------

def bf16_to_f32(h: int) -> float:
    return float(lib().ora_bf16_to_f32(h))


def f32_to_bf16(f: float) -> int:
    return int(lib().ora_f32_to_bf16(f))


def e2m1_decode(code: int) -> float:
    return float(lib().ora_e2m1_decode(code))


def e2m1_encode(v: float) -> int:
    return int(lib().ora_e2m1_encode(v))


def e4m3_decode(b: int) -> float:
    return float(lib().ora_e4m3_decode(b))


def e4m3_encode(v: float) -> int:
    return int(lib().ora_e4m3_encode(v))


def e2m1_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint8)
    lib().ora_e2m1_encode_array(v, v.size, out)
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint8)
    lib().ora_e4m3_encode_array(v, v.size, out)
    return out


def f32_to_bf16_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint16)
    lib().ora_f32_to_bf16_array(v, v.size, out)
    return out


def global_scale(amax: float) -> float:
    return float(lib().ora_global_scale(amax))


def alpha(gsf_x: float, gsf_w: float) -> float:
    return float(lib().ora_alpha(gsf_x, gsf_w))


def hadamard_scale(g: int) -> float:
    return float(lib().ora_hadamard_scale(g))


# --------------------------------------------------------------------------
# tensors (numpy in, numpy out)
# --------------------------------------------------------------------------

def _u16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 tensors are passed as uint16 bit patterns"
    return x


def amax_bf16(x: np.ndarray) -> float:
    x = _u16(x)
    return float(lib().ora_amax_bf16(x.reshape(-1), x.size))


def scale_bytes(rows: int, K: int) -> int:
    return int(lib().ora_scale_bytes(rows, K))


def scale_offset(r: int, c: int, K: int) -> int:
    return int(lib().ora_scale_offset(r, c, K))


def scale_swizzle(sf_lin: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.empty(scale_bytes(rows, K), dtype=np.uint8)
    lib().ora_scale_swizzle(np.ascontiguousarray(sf_lin, dtype=np.uint8).reshape(-1), rows, K, out)
    return out


def scale_unswizzle(sf: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.empty((rows, K // 16), dtype=np.uint8)
    lib().ora_scale_unswizzle(np.ascontiguousarray(sf, dtype=np.uint8).reshape(-1), rows, K,
                              out.reshape(-1))
    return out


def quantize_rows(x: np.ndarray, gsf: float):
    """Block quantize with a given global scale -> (packed [R,K/2], sf_lin [R,K/16])."""
    x = _u16(x)
    R, K = x.shape
    packed = np.empty((R, K // 2), dtype=np.uint8)
    sf_lin = np.empty((R, K // 16), dtype=np.uint8)
    lib().ora_quantize_rows(x.reshape(-1), R, K, np.float32(gsf), packed.reshape(-1),
                            sf_lin.reshape(-1))
    return packed, sf_lin


def quantize(x: np.ndarray, gsf: float | None = None):
    """Full quantizer -> (packed [R,K/2], sf in the 128x4 layout, gsf used).

    ``gsf=None`` is the dynamic scale (amax over the whole tensor)."""
    x = _u16(x)
    R, K = x.shape
    packed = np.empty((R, K // 2), dtype=np.uint8)
    sf = np.empty(scale_bytes(R, K), dtype=np.uint8)
    scratch = np.empty(max(R * K // 16, 1), dtype=np.uint8)
    g = lib().ora_quantize(x.reshape(-1), R, K, np.float32(-1.0 if gsf is None else gsf),
                           packed.reshape(-1), sf, scratch)
    return packed, sf, float(np.float32(g))


def hadamard_rotate(x: np.ndarray, g: int) -> np.ndarray:
    x = _u16(x)
    R, K = x.shape
    y = np.empty_like(x)
    lib().ora_hadamard_rotate(x.reshape(-1), R, K, int(g), y.reshape(-1))
    return y


def dequantize(packed: np.ndarray, sf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """fp64 [rows, K] = E2M1(code) * E4M3(block scale); the global scale is not applied."""
    out = np.empty((rows, K), dtype=np.float64)
    lib().ora_dequantize(np.ascontiguousarray(packed).reshape(-1), np.ascontiguousarray(sf).reshape(-1),
                         rows, K, out.reshape(-1))
    return out


def dequantize_bf16(packed: np.ndarray, sf: np.ndarray, rows: int, K: int, gsf: float) -> np.ndarray:
    """bf16 bits [rows, K] = RNE_bf16(fp32(E2M1(code) * E4M3(scale)) / gsf)."""
    out = np.empty((rows, K), dtype=np.uint16)
    lib().ora_dequantize_bf16(np.ascontiguousarray(packed).reshape(-1),
                              np.ascontiguousarray(sf).reshape(-1), rows, K, np.float32(gsf),
                              out.reshape(-1))
    return out


def int8_quantize_rows(x: np.ndarray):
    """bf16 [R, K] -> (int8 codes [R, K], fp32 row scales [R]) (per-row amax / 127)."""
    x = _u16(x)
    R, K = x.shape
    q = np.empty((R, K), dtype=np.int8)
    s = np.empty(R, dtype=np.float32)
    lib().ora_int8_quantize_rows(x.reshape(-1), R, K, q.reshape(-1), s)
    return q, s


def int8_gemm_f64(qx: np.ndarray, sx: np.ndarray, qw: np.ndarray, sw: np.ndarray,
                  bias: np.ndarray | None = None, rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 y[rows, N] = s_x[m] s_w[n] sum_k qx qw + bias."""
    M, K = qx.shape
    N = qw.shape[0]
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = M if rows_arr is None else rows_arr.size
    y = np.empty((n_rows, N), dtype=np.float64)
    bias_arr = None if bias is None else np.ascontiguousarray(_u16(bias).reshape(-1))
    lib().ora_int8_gemm_f64(np.ascontiguousarray(qx).reshape(-1), np.ascontiguousarray(sx, dtype=np.float32),
                            np.ascontiguousarray(qw).reshape(-1), np.ascontiguousarray(sw, dtype=np.float32),
                            N, K, None if bias_arr is None else bias_arr.ctypes.data,
                            None if rows_arr is None else rows_arr.ctypes.data, n_rows, y.reshape(-1))
    return y


def gemm_f64(a: np.ndarray, sfa: np.ndarray, b: np.ndarray, sfb: np.ndarray, M: int, N: int,
             K: int, alpha_: float, bias: np.ndarray | None = None,
             rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 y[rows, N] = alpha * deq(a) deq(b)^T + bias (rows: subset of 0..M-1)."""
    a = np.ascontiguousarray(a).reshape(-1)
    b = np.ascontiguousarray(b).reshape(-1)
    sfa = np.ascontiguousarray(sfa).reshape(-1)
    sfb = np.ascontiguousarray(sfb).reshape(-1)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = M if rows_arr is None else rows_arr.size
    y = np.empty((n_rows, N), dtype=np.float64)
    bias_arr = None if bias is None else _u16(bias).reshape(-1)
    lib().ora_gemm_f64(a, sfa, b, sfb, N, K, np.float32(alpha_),
                       None if bias_arr is None else bias_arr.ctypes.data,
                       None if rows_arr is None else rows_arr.ctypes.data, n_rows, y.reshape(-1))
    return y


def linear(x: np.ndarray, w_packed: np.ndarray, w_sf: np.ndarray, gsf_w: float, N: int,
           bias: np.ndarray | None = None, gsf_x: float | None = None, rotate_group: int = 0,
           rows: np.ndarray | None = None):
    """The whole path on bf16 x [M, K]: rotate (optional) -> quantize -> fp64 GEMM.

    The weight must already be rotated and packed.  Returns (y64 [rows, N], packed_x,
    sf_x, gsf_x used, alpha)."""
    x = _u16(x)
    M, K = x.shape
    xr = hadamard_rotate(x, rotate_group) if rotate_group else x
    xp, xsf, g = quantize(xr, gsf_x)
    al = alpha(g, gsf_w)
    y = gemm_f64(xp, xsf, w_packed, w_sf, M, N, K, al, bias, rows)
    return y, xp, xsf, g, al
