"""CPU oracle for the Q4_0 and super-block K-quant ("ksb") formats.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.  The CUDA library and its
Python binding never import it, and it imports nothing from them.

The arithmetic lives in ``gq_oracle.c`` (plain C, gcc, no fast-math); this
module only builds that file and marshals numpy arrays through ctypes.
Sources: the Q4_0 chapter ("GGUF 量化内幕 第4章", sections 4.1-4.5) and the
K-quants super-block post ("GGUF K-quants", section "套娃").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FMT_Q4_0 = 0
FMT_KSB = 1
F32, F16, BF16 = 0, 1, 2
RULE_ABSMAX7 = 0
RULE_LLAMA = 1
NONFINITE = 1
RANGE = 2

Q4_0_BLOCK, Q4_0_BYTES = 32, 18
KSB_BLOCK, KSB_BYTES = 256, 138


def build(force: bool = False) -> str:
    """Compile gq_oracle.c with gcc into liboracle.so (IEEE, no contraction)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)
            and os.path.getmtime(_LIB) >= os.path.getmtime(os.path.join(_HERE, "gq_oracle.h"))):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
           "-fexcess-precision=standard", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", _LIB, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, vp, dp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
        L.orc_f32_to_f16.argtypes = [ctypes.c_float]
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f32.restype = ctypes.c_float
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_f32_to_f16_array.argtypes = [vp, i64, vp]
        L.orc_f16_to_f32_array.argtypes = [vp, i64, vp]
        L.orc_q4_0_bytes.argtypes = [i64]
        L.orc_q4_0_bytes.restype = i64
        L.orc_ksb_bytes.argtypes = [i64]
        L.orc_ksb_bytes.restype = i64
        L.orc_quantize_q4_0.argtypes = [vp, i64, vp, ctypes.c_int]
        L.orc_quantize_q4_0.restype = ctypes.c_int
        L.orc_quantize_ksb.argtypes = [vp, i64, vp]
        L.orc_quantize_ksb.restype = ctypes.c_int
        L.orc_ksb_scale_step.argtypes = [vp, vp, vp]
        L.orc_dequantize_q4_0.argtypes = [vp, i64, vp]
        L.orc_dequantize_ksb.argtypes = [vp, i64, vp]
        L.orc_gemm.argtypes = [ctypes.c_int, vp, i64, i64, vp, ctypes.c_int, i64, dp, dp]
        L.orc_gemm_rows.argtypes = [ctypes.c_int, vp, i64, i64, vp, ctypes.c_int, i64,
                                    vp, i64, dp, dp]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_threads.argtypes = [ctypes.c_int]
        L.orc_set_threads.restype = None
        L.orc_tiled_bytes.argtypes = [ctypes.c_int, i64, i64]
        L.orc_tiled_bytes.restype = i64
        L.orc_repack.argtypes = [ctypes.c_int, vp, i64, i64, vp]
        L.orc_repack.restype = ctypes.c_int
        L.orc_unrepack.argtypes = [ctypes.c_int, vp, i64, i64, vp]
        L.orc_unrepack.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# --- scalar / array converters ------------------------------------------------

def f32_to_f16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, dtype=np.uint16)
    lib().orc_f32_to_f16_array(_ptr(x), x.size, _ptr(out))
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16).ravel()
    out = np.empty(h.size, dtype=np.float32)
    lib().orc_f16_to_f32_array(_ptr(h), h.size, _ptr(out))
    return out


def f32_to_bf16_bits(v: float) -> int:
    return int(lib().orc_f32_to_bf16(float(v)))


def bf16_bits_to_f32(h: int) -> float:
    return float(lib().orc_bf16_to_f32(int(h)))


# --- formats -------------------------------------------------------------------

def q4_0_bytes(n: int) -> int:
    return int(lib().orc_q4_0_bytes(n))


def ksb_bytes(n: int) -> int:
    return int(lib().orc_ksb_bytes(n))


def quantize_q4_0(x, rule: int = RULE_ABSMAX7):
    """fp32 values (n % 32 == 0) -> (uint8 bytes, status flags)."""
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.zeros(q4_0_bytes(x.size), dtype=np.uint8)
    flags = lib().orc_quantize_q4_0(_ptr(x), x.size, _ptr(out), rule)
    if flags < 0:
        raise ValueError("n must be a multiple of 32")
    return out, flags


def quantize_ksb(x):
    """fp32 values (n % 256 == 0) -> (uint8 bytes, status flags)."""
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.zeros(ksb_bytes(x.size), dtype=np.uint8)
    flags = lib().orc_quantize_ksb(_ptr(x), x.size, _ptr(out))
    if flags < 0:
        raise ValueError("n must be a multiple of 256")
    return out, flags


def quantize(fmt: int, x):
    return quantize_q4_0(x) if fmt == FMT_Q4_0 else quantize_ksb(x)


def ksb_scale_step(d16_bits):
    """Eight FP16 sub-scales (bit patterns) -> (super-scale bits, int8 codes)."""
    d = np.ascontiguousarray(d16_bits, dtype=np.uint16)
    assert d.size == 8
    s = np.zeros(1, dtype=np.uint16)
    q = np.zeros(8, dtype=np.int8)
    lib().orc_ksb_scale_step(_ptr(d), _ptr(s), _ptr(q))
    return int(s[0]), q


def dequantize_q4_0(q, n: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).ravel()
    assert q.size >= q4_0_bytes(n)
    out = np.empty(n, dtype=np.float32)
    lib().orc_dequantize_q4_0(_ptr(q), n, _ptr(out))
    return out


def dequantize_ksb(q, n: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).ravel()
    assert q.size >= ksb_bytes(n)
    out = np.empty(n, dtype=np.float32)
    lib().orc_dequantize_ksb(_ptr(q), n, _ptr(out))
    return out


def dequantize(fmt: int, q, n: int) -> np.ndarray:
    return dequantize_q4_0(q, n) if fmt == FMT_Q4_0 else dequantize_ksb(q, n)


def _x_code(X: np.ndarray, xt: int | None):
    if xt is not None:
        return xt
    if X.dtype == np.float32:
        return F32
    if X.dtype == np.float16:
        return F16
    raise TypeError("pass bfloat16 activations as uint16 bit patterns with xt=BF16")


def gemm(fmt: int, W, M: int, K: int, X, xt: int | None = None):
    """Y[b, m] = sum_k What[m, k] X[b, k] in fp64, plus sum_k |What||X|.

    X: [B, K] float32 / float16, or uint16 bfloat16 bits with xt=BF16.
    Returns (Y, bound), both float64 [B, M]."""
    W = np.ascontiguousarray(W, dtype=np.uint8).ravel()
    X = np.ascontiguousarray(X)
    if X.ndim == 1:
        X = X[None, :]
    B = X.shape[0]
    assert X.shape[1] == K
    Y = np.empty((B, M), dtype=np.float64)
    bound = np.empty((B, M), dtype=np.float64)
    lib().orc_gemm(fmt, _ptr(W), M, K, _ptr(X), _x_code(X, xt), B, _ptr(Y), _ptr(bound))
    return Y, bound


def gemm_rows(fmt: int, W, M: int, K: int, X, rows, xt: int | None = None):
    """As gemm(), for the listed rows only: returns ([B, len(rows)], bound)."""
    W = np.ascontiguousarray(W, dtype=np.uint8).ravel()
    X = np.ascontiguousarray(X)
    if X.ndim == 1:
        X = X[None, :]
    B = X.shape[0]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.empty((B, rows.size), dtype=np.float64)
    bound = np.empty((B, rows.size), dtype=np.float64)
    lib().orc_gemm_rows(fmt, _ptr(W), M, K, _ptr(X), _x_code(X, xt), B,
                        _ptr(rows), rows.size, _ptr(Y), _ptr(bound))
    return Y, bound


def tiled_bytes(fmt: int, M: int, K: int) -> int:
    """Bytes of the tiled storage of an M x K matrix (-1: K not a whole number
    of units)."""
    return int(lib().orc_tiled_bytes(fmt, M, K))


def repack(fmt: int, W, M: int, K: int) -> np.ndarray:
    """Canonical packed rows -> tiled storage (layout in gq_oracle.h)."""
    W = np.ascontiguousarray(W, dtype=np.uint8).ravel()
    n = tiled_bytes(fmt, M, K)
    if n < 0:
        raise ValueError("K must be a multiple of 64 (Q4_0) or 256 (ksb)")
    out = np.zeros(n, dtype=np.uint8)
    lib().orc_repack(fmt, _ptr(W), M, K, _ptr(out))
    return out


def unrepack(fmt: int, T, M: int, K: int) -> np.ndarray:
    """Tiled storage -> canonical packed rows (the inverse of repack)."""
    T = np.ascontiguousarray(T, dtype=np.uint8).ravel()
    rb = q4_0_bytes(K) if fmt == FMT_Q4_0 else ksb_bytes(K)
    out = np.zeros(M * rb, dtype=np.uint8)
    if lib().orc_unrepack(fmt, _ptr(T), M, K, _ptr(out)) < 0:
        raise ValueError("K must be a multiple of 64 (Q4_0) or 256 (ksb)")
    return out


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_threads(n: int) -> None:
    """Threads of the oracle's parallel loops from now on (timing only)."""
    lib().orc_set_threads(int(n))
