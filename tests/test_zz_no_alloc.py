"""q4_gemv_noalloc: the GEMV for callers that cannot allocate device memory.

Such callers (a plugin whose host application owns every device allocation, a
runtime whose memory budget is fixed after start-up, a latency-critical path that
must not call cudaMalloc) cannot pass a workspace, so this entry point keeps its
split-K scratch in a fixed 1 MiB device array inside the library. The test calls
it through the C ABI, twice in a row, and checks each result against q4_gemv
(the entry point with a caller workspace) within the parity tolerance
|y - y_ref| <= 1e-4 * sum|w x| + 1e-6. It sits in a file collected last and also
passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from quantized_decode_q4_b200 import q4, synth

pytestmark = pytest.mark.gpu


def _noalloc():
    fn = q4.lib().q4_gemv_noalloc
    fn.argtypes = [ctypes.POINTER(q4.q4_matrix), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


@pytest.mark.parametrize("shape", [(1024, 4096), (4096, 14336), (1408, 512), (50257, 768)])
def test_noalloc_matches_workspace_entry_point(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    n, k = shape
    fn = _noalloc()
    w = synth.matrix(41, n, n, k, synth.WEIGHT_STD, device="cuda")
    m = q4.pack(w)
    del w
    x = synth.normal(41, n + 1, 0, k, 1.0, device="cuda")
    y_ref = q4.gemv(m, x)                       # existing entry point, caller workspace
    w_hat = q4.dequant(m)
    abs_sum = (w_hat.double().abs() @ x.double().abs())
    del w_hat
    cm = m.c()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y = torch.full((n,), float("nan"), device="cuda")
        status = fn(ctypes.byref(cm), x.data_ptr(), y.data_ptr(), stream)
        assert status == 0, q4.status_string(status)
        torch.cuda.synchronize()
        err = (y.double() - y_ref.double()).abs()
        bound = 1e-4 * abs_sum + 1e-6
        assert bool(torch.all(err <= bound)), f"call {call}: max err {err.max().item()}"


def test_noalloc_rejects_matrices_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    fn = _noalloc()
    n, k = 64, 1 << 25   # split-K partial sums of about 2 MiB, beyond the 1 MiB array
    assert q4.workspace_bytes(n, k, 1) > (1 << 20)
    m = q4.q4_matrix(256, 256, n, k)  # never dereferenced: rejected before any launch
    assert fn(ctypes.byref(m), 256, 256, None) == 3
