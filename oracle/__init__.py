"""Q4_0 decode oracle: ctypes wrapper over the plain C reference in q4_oracle.c.

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg (``bench.py --impl reference`` and the
``cpu_baseline`` object) may import this package. The product package
``quantized_decode_q4_b200`` never imports it, and this package imports nothing
from the product.

Every function follows the pages on Q4 decode:
  * "MicroLLM Lab" (sitech.ge), "Seven models, all in Q4": weights stored at
    4 bits per parameter;
  * "Llamas on the Web" (gist.science summary of arXiv 2605.20706), section
    "Design di Shader Consapevole della Quantizzazione": packed quantised words,
    dequantised inside the matrix-vector product at decode time.
The Q4_0 block layout (32 weights, binary16 d, w = d*(q-8), 18 bytes) and the
readings of what the pages leave open are stated in q4_oracle.c's header.

Pins: every function here is checked by tests/test_oracle_*.py against values
that do not come from this code (hand-derived golden blocks, numpy's binary16
conversion, exact rational arithmetic, closed forms). The layer-stack
throughput has no value on the pages: "parity unpinned" for that figure only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_q4.so")

QK = 32
BLOCK_BYTES = 18

CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile q4_oracle.c with gcc (no FMA contraction) and return the .so path."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call(["gcc", *CFLAGS, src, "-o", out, "-lm"])
    return out


_lib = None


def _bind(lib):
    c = ctypes
    u8p, f32p, f64p, u16p = (c.POINTER(c.c_uint8), c.POINTER(c.c_float),
                             c.POINTER(c.c_double), c.POINTER(c.c_uint16))
    lib.oracle_f32_to_f16.argtypes = [c.c_float]
    lib.oracle_f32_to_f16.restype = c.c_uint16
    lib.oracle_f16_to_f32.argtypes = [c.c_uint16]
    lib.oracle_f16_to_f32.restype = c.c_float
    lib.oracle_q4_pack.argtypes = [f32p, c.c_int64, c.c_int64, u8p]
    lib.oracle_q4_dequant.argtypes = [u8p, c.c_int64, c.c_int64, f32p]
    lib.oracle_q4_gemv.argtypes = [u8p, c.c_int64, c.c_int64, f32p, f64p, f64p]
    lib.oracle_q4_gemv_batched.argtypes = [u8p, c.c_int64, c.c_int64, f32p, c.c_int64,
                                           f64p, f64p]
    lib.oracle_blocks_to_planes.argtypes = [u8p, c.c_int64, c.c_int64, u8p, u16p]
    for fn in ("oracle_q4_pack", "oracle_q4_dequant", "oracle_q4_gemv",
               "oracle_q4_gemv_batched", "oracle_blocks_to_planes"):
        getattr(lib, fn).restype = c.c_int
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check_k(k: int):
    if k % QK != 0:
        raise ValueError(f"k={k} is not a multiple of {QK}")


def f32_to_f16(values, lib=None) -> np.ndarray:
    """binary32 -> binary16 bits (round to nearest even), element by element."""
    lib = lib or load()
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    return np.array([lib.oracle_f32_to_f16(float(x)) for x in v], dtype=np.uint16)


def f16_to_f32(bits, lib=None) -> np.ndarray:
    """binary16 bits -> binary32 values (exact)."""
    lib = lib or load()
    b = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.oracle_f16_to_f32(int(h)) for h in b], dtype=np.float32)


def q4_pack(w: np.ndarray, lib=None) -> np.ndarray:
    """Row-major binary32 W[n][k] -> Q4_0 blocks, uint8 array of shape [n, k/32, 18]."""
    lib = lib or load()
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    _check_k(k)
    out = np.zeros((n, k // QK, BLOCK_BYTES), dtype=np.uint8)
    rc = lib.oracle_q4_pack(_ptr(w, ctypes.c_float), n, k, _ptr(out, ctypes.c_uint8))
    if rc:
        raise ValueError("oracle_q4_pack rejected its arguments")
    return out


def q4_dequant(blocks: np.ndarray, n: int, k: int, lib=None) -> np.ndarray:
    """Q4_0 blocks -> binary32 W_hat[n][k] (exact)."""
    lib = lib or load()
    _check_k(k)
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    assert blocks.size == n * (k // QK) * BLOCK_BYTES
    out = np.zeros((n, k), dtype=np.float32)
    lib.oracle_q4_dequant(_ptr(blocks, ctypes.c_uint8), n, k, _ptr(out, ctypes.c_float))
    return out


def q4_gemv(blocks: np.ndarray, n: int, k: int, x: np.ndarray, lib=None):
    """y = W_hat x in binary64 (index-order sum). Returns (y, abs_sum), both float64 [n]."""
    lib = lib or load()
    _check_k(k)
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    assert x.size == k and blocks.size == n * (k // QK) * BLOCK_BYTES
    y = np.zeros(n, dtype=np.float64)
    s = np.zeros(n, dtype=np.float64)
    lib.oracle_q4_gemv(_ptr(blocks, ctypes.c_uint8), n, k, _ptr(x, ctypes.c_float),
                       _ptr(y, ctypes.c_double), _ptr(s, ctypes.c_double))
    return y, s


def q4_gemv_batched(blocks: np.ndarray, n: int, k: int, X: np.ndarray, lib=None):
    """Y[t] = W_hat X[t] for every token t. Returns (Y, abs_sum), float64 [b, n]."""
    lib = lib or load()
    _check_k(k)
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    X = np.ascontiguousarray(X, dtype=np.float32)
    b = X.shape[0]
    assert X.shape == (b, k)
    Y = np.zeros((b, n), dtype=np.float64)
    S = np.zeros((b, n), dtype=np.float64)
    lib.oracle_q4_gemv_batched(_ptr(blocks, ctypes.c_uint8), n, k, _ptr(X, ctypes.c_float),
                               b, _ptr(Y, ctypes.c_double), _ptr(S, ctypes.c_double))
    return Y, S


def blocks_to_planes(blocks: np.ndarray, n: int, k: int, lib=None):
    """Q4_0 blocks -> (qs uint8 [n, k/2], d uint16 [n, k/32]) with the same bytes."""
    lib = lib or load()
    _check_k(k)
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    qs = np.zeros((n, k // 2), dtype=np.uint8)
    d = np.zeros((n, k // QK), dtype=np.uint16)
    lib.oracle_blocks_to_planes(_ptr(blocks, ctypes.c_uint8), n, k,
                                _ptr(qs, ctypes.c_uint8), _ptr(d, ctypes.c_uint16))
    return qs, d


def gemv_within_tolerance(y_test, y_ref, abs_sum, rel=1e-4, abs_tol=1e-6):
    """Per-element GEMV acceptance: |y - y_ref| <= rel * sum|w_i x_i| + abs_tol."""
    y_test = np.asarray(y_test, dtype=np.float64)
    return np.abs(y_test - y_ref) <= rel * abs_sum + abs_tol
