"""ctypes binding of libq4_b200.so (the C ABI in include/q4.h).

Argument marshalling only: tensors become device pointers, torch's current
stream becomes the cudaStream_t, status codes become exceptions. Every step of
the computation runs in the library's CUDA kernels; there is no fallback. If the
shared library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libq4_b200.so")

QK = 32
MAX_BATCH = 16
MAX_GROUP = 8

STATUS = {0: "ok", 1: "invalid argument", 2: "misaligned pointer",
          3: "workspace missing or too small", 4: "unsupported (batch or device)",
          5: "CUDA error", 6: "device wait timed out"}


class Q4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class q4_matrix(ctypes.Structure):
    _fields_ = [("qs", ctypes.c_void_p), ("d", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64)]


class q4_stack(ctypes.Structure):
    _fields_ = [("count", ctypes.c_int), ("mats", ctypes.POINTER(q4_matrix)),
                ("x", ctypes.POINTER(ctypes.c_void_p)), ("y", ctypes.POINTER(ctypes.c_void_p)),
                ("group", ctypes.POINTER(ctypes.c_int))]


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantized_decode_q4_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        vp, i64, sz = c.c_void_p, c.c_int64, c.c_size_t
        mp = c.POINTER(q4_matrix)
        sp = c.POINTER(q4_stack)
        sig = {
            "q4_plane_bytes": ([i64, i64, c.POINTER(sz), c.POINTER(sz)], c.c_int),
            "q4_pack": ([vp, mp, vp], c.c_int),
            "q4_dequant": ([mp, vp, vp], c.c_int),
            "q4_workspace_bytes": ([i64, i64, c.c_int], sz),
            "q4_workspace_init": ([vp, sz, vp], c.c_int),
            "q4_workspace_status": ([vp, vp], c.c_int),
            "q4_gemv": ([mp, vp, vp, vp, sz, vp], c.c_int),
            "q4_gemv_batched": ([mp, vp, c.c_int, vp, vp, sz, vp], c.c_int),
            "q4_stack_workspace_bytes": ([sp, c.c_int], sz),
            "q4_layer_stack": ([sp, c.c_int, vp, sz, vp], c.c_int),
            "q4_stack_graph_create": ([sp, c.c_int, vp, sz, vp, c.POINTER(vp)], c.c_int),
            "q4_graph_launch": ([vp, vp], c.c_int),
            "q4_graph_destroy": ([vp], c.c_int),
            "q4_blocks_to_planes": ([vp, i64, i64, vp, vp], c.c_int),
            "q4_planes_to_blocks": ([vp, vp, i64, i64, vp], c.c_int),
            "q4_status_string": ([c.c_int], c.c_char_p),
            "q4_launch_count": ([], c.c_uint64),
            "q4_last_cuda_error": ([], c.c_char_p),
            "q4_debug_check_b1": ([c.POINTER(i64), c.POINTER(i64), c.c_int, c.c_int, c.c_int], c.c_int),
            "q4_gemv_noalloc": ([mp, vp, vp, vp], c.c_int),
            "q4_noalloc_status": ([vp], c.c_int),
            "q4_debug_plan_info": ([c.POINTER(i64), c.POINTER(i64), c.c_int, c.c_int,
                                    c.POINTER(i64)], c.c_int),
            "q4_debug_check_unpack": ([c.c_uint64, i64], i64),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        if status == 5:
            where = f"{where} [{lib().q4_last_cuda_error().decode()}]"
        raise Q4Error(status, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


# ---------------------------------------------------------------------------
# matrices
# ---------------------------------------------------------------------------

def plane_bytes(n: int, k: int):
    qs, d = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().q4_plane_bytes(n, k, ctypes.byref(qs), ctypes.byref(d)), "q4_plane_bytes")
    return qs.value, d.value


class Q4Matrix:
    """A Q4_0 matrix in planes layout, owning its two device tensors."""

    def __init__(self, n: int, k: int, device="cuda", qs=None, d=None):
        qs_b, d_b = plane_bytes(n, k)
        self.n, self.k = n, k
        self.qs = qs if qs is not None else torch.empty(qs_b, dtype=torch.uint8, device=device)
        self.d = d if d is not None else torch.zeros(d_b // 2, dtype=torch.int16, device=device)
        assert self.qs.numel() >= qs_b and self.d.numel() * 2 >= d_b

    def c(self) -> q4_matrix:
        return q4_matrix(self.qs.data_ptr(), self.d.data_ptr(), self.n, self.k)

    @property
    def nbytes(self) -> int:
        return self.n * self.k * 18 // 32

    def qs_plane(self) -> torch.Tensor:
        return self.qs[: self.n * self.k // 2].view(self.n, self.k // 2)

    def d_plane(self) -> torch.Tensor:
        return self.d[: self.n * self.k // QK].view(self.n, self.k // QK)


def pack(w: torch.Tensor, out: Q4Matrix | None = None, stream=None) -> Q4Matrix:
    """Quantise a row-major binary32 device matrix [n][k] to Q4_0 planes."""
    assert w.dtype == torch.float32 and w.is_cuda and w.is_contiguous() and w.dim() == 2
    n, k = w.shape
    m = out if out is not None else Q4Matrix(n, k, device=w.device)
    cm = m.c()
    _check(lib().q4_pack(_ptr(w), ctypes.byref(cm), _stream(stream)), "q4_pack")
    return m


def dequant(m: Q4Matrix, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    o = out if out is not None else torch.empty(m.n, m.k, dtype=torch.float32, device=m.qs.device)
    cm = m.c()
    _check(lib().q4_dequant(ctypes.byref(cm), _ptr(o), _stream(stream)), "q4_dequant")
    return o


# ---------------------------------------------------------------------------
# workspace
# ---------------------------------------------------------------------------

def workspace_bytes(n: int, k: int, b: int = 1) -> int:
    v = lib().q4_workspace_bytes(n, k, b)
    if v == 0:
        raise Q4Error(1, "q4_workspace_bytes")
    return v


def workspace(nbytes: int, device="cuda", stream=None) -> torch.Tensor:
    """A zero-initialised workspace (torch allocations are 512-byte aligned)."""
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    _check(lib().q4_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "q4_workspace_init")
    return ws


def workspace_init(ws: torch.Tensor, stream=None) -> None:
    """Zero a workspace again (clears a recorded timeout)."""
    _check(lib().q4_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "q4_workspace_init")


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    return lib().q4_workspace_status(_ptr(ws), _stream(stream))


# ---------------------------------------------------------------------------
# products
# ---------------------------------------------------------------------------

def gemv(m: Q4Matrix, x: torch.Tensor, y: torch.Tensor | None = None,
         ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = W x for one token (x binary32 [k] on the device)."""
    y = y if y is not None else torch.empty(m.n, dtype=torch.float32, device=x.device)
    ws = ws if ws is not None else workspace(workspace_bytes(m.n, m.k, 1), x.device, stream)
    cm = m.c()
    _check(lib().q4_gemv(ctypes.byref(cm), _ptr(x), _ptr(y), _ptr(ws), ws.numel(),
                         _stream(stream)), "q4_gemv")
    return y


def gemv_batched(m: Q4Matrix, X: torch.Tensor, Y: torch.Tensor | None = None,
                 ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y[t] = W X[t] for t < b (X binary32 [b][k] on the device, 1 <= b <= 16)."""
    b = X.shape[0]
    Y = Y if Y is not None else torch.empty(b, m.n, dtype=torch.float32, device=X.device)
    ws = ws if ws is not None else workspace(workspace_bytes(m.n, m.k, b), X.device, stream)
    cm = m.c()
    _check(lib().q4_gemv_batched(ctypes.byref(cm), _ptr(X), b, _ptr(Y), _ptr(ws), ws.numel(),
                                 _stream(stream)), "q4_gemv_batched")
    return Y


class Stack:
    """A decode step: GEMVs with dependency groups, inputs and outputs."""

    def __init__(self, mats, xs, ys, groups):
        assert len(mats) == len(xs) == len(ys) == len(groups)
        self.mats, self.xs, self.ys, self.groups = list(mats), list(xs), list(ys), list(groups)
        cnt = len(mats)
        self._mats = (q4_matrix * cnt)(*[m.c() for m in mats])
        self._x = (ctypes.c_void_p * cnt)(*[x.data_ptr() for x in xs])
        self._y = (ctypes.c_void_p * cnt)(*[y.data_ptr() for y in ys])
        self._g = (ctypes.c_int * cnt)(*groups)
        self.c = q4_stack(cnt, self._mats, self._x, self._y, self._g)

    def workspace_bytes(self, b: int) -> int:
        v = lib().q4_stack_workspace_bytes(ctypes.byref(self.c), b)
        if v == 0:
            raise Q4Error(1, "q4_stack_workspace_bytes")
        return v


def layer_stack(stack: Stack, b: int, ws: torch.Tensor, stream=None):
    _check(lib().q4_layer_stack(ctypes.byref(stack.c), b, _ptr(ws), ws.numel(), _stream(stream)),
           "q4_layer_stack")


class Graph:
    """One captured decode step, replayed with a single call."""

    def __init__(self, stack: Stack, b: int, ws: torch.Tensor, stream):
        self.stack, self.ws = stack, ws  # keep the buffers alive
        h = ctypes.c_void_p()
        _check(lib().q4_stack_graph_create(ctypes.byref(stack.c), b, _ptr(ws), ws.numel(),
                                           _stream(stream), ctypes.byref(h)),
               "q4_stack_graph_create")
        self.h = h

    def launch(self, stream=None):
        _check(lib().q4_graph_launch(self.h, _stream(stream)), "q4_graph_launch")

    def close(self):
        if self.h:
            _check(lib().q4_graph_destroy(self.h), "q4_graph_destroy")
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# host helpers
# ---------------------------------------------------------------------------

def blocks_to_planes(blocks: np.ndarray, n: int, k: int):
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    qs = np.zeros((n, k // 2), np.uint8)
    d = np.zeros((n, k // QK), np.uint16)
    _check(lib().q4_blocks_to_planes(blocks.ctypes.data, n, k, qs.ctypes.data, d.ctypes.data),
           "q4_blocks_to_planes")
    return qs, d


def planes_to_blocks(qs: np.ndarray, d: np.ndarray, n: int, k: int) -> np.ndarray:
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    d = np.ascontiguousarray(d, dtype=np.uint16)
    out = np.zeros((n, k // QK, 18), np.uint8)
    _check(lib().q4_planes_to_blocks(qs.ctypes.data, d.ctypes.data, n, k, out.ctypes.data),
           "q4_planes_to_blocks")
    return out


def gemv_noalloc(m: Q4Matrix, x: torch.Tensor, y: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """y = W x for one token with the library's fixed scratch array (no workspace)."""
    y = y if y is not None else torch.empty(m.n, dtype=torch.float32, device=x.device)
    cm = m.c()
    _check(lib().q4_gemv_noalloc(ctypes.byref(cm), _ptr(x), _ptr(y), _stream(stream)),
           "q4_gemv_noalloc")
    return y


def noalloc_status(stream=None) -> int:
    """Q4_ERR_TIMEOUT (6) if a q4_gemv_noalloc wait gave up since the last call, else 0."""
    return lib().q4_noalloc_status(_stream(stream))


def launch_count() -> int:
    return lib().q4_launch_count()


def status_string(s: int) -> str:
    return lib().q4_status_string(s).decode()


def check_b1(shapes, num_sms: int = 148, b: int = 1) -> int:
    """Host replay of the CUDA-core launch plan for b tokens (0 when every check
    holds)."""
    n = (ctypes.c_int64 * len(shapes))(*[s[0] for s in shapes])
    k = (ctypes.c_int64 * len(shapes))(*[s[1] for s in shapes])
    return lib().q4_debug_check_b1(n, k, len(shapes), b, num_sms)


def plan_info(shapes, b: int = 1) -> dict:
    """The CUDA-core plan of one launch for b tokens on a 148-SM B200."""
    n = (ctypes.c_int64 * len(shapes))(*[s[0] for s in shapes])
    k = (ctypes.c_int64 * len(shapes))(*[s[1] for s in shapes])
    out = (ctypes.c_int64 * (4 + len(shapes)))()
    _check(lib().q4_debug_plan_info(n, k, len(shapes), b, out), "q4_debug_plan_info")
    return {"pieces": out[0], "smem": out[1], "ws_bytes": out[2], "slots": out[3],
            "splits": [out[4 + i] for i in range(len(shapes))]}


def check_unpack(seed: int = 1, count: int = 100000) -> int:
    return lib().q4_debug_check_unpack(seed, count)
