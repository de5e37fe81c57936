"""q4_gemv_noalloc: the GEMV for callers that cannot allocate device memory.

Such callers (a plugin whose host application owns every device allocation, a
runtime whose memory budget is fixed after start-up, a latency-critical path that
must not call cudaMalloc) cannot pass a workspace, so this entry point keeps its
split-K scratch in a fixed 1 MiB device array inside the library. The test calls
it through the C ABI, twice in a row per shape, and checks each result
bit for bit against q4_gemv (the entry point with a caller workspace: same kernel,
same plan) and, on sampled rows, against the oracle within the parity tolerance
|y - y_ref| <= 1e-4 * sum|w x| + 1e-6. Shapes alternate between a narrow matrix
whose K is split across CTAs (so the shared array's tickets and partial sums are
used) and others, larger before smaller, so a later call runs on the contents the
earlier one left behind. It sits in a file collected last and also passes on its
own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_util import assert_gemv_close, oracle_rows, sample_rows
from quantized_decode_q4_b200 import q4, synth

pytestmark = pytest.mark.gpu

# (2, 131072): K split across CTAs (tickets and partials in the array);
# (3, 28672) and (17, 4096): smaller split layouts after a larger one
SHAPES = [(4096, 14336), (2, 131072), (1408, 512), (3, 28672), (50257, 768), (17, 4096)]


def _noalloc():
    fn = q4.lib().q4_gemv_noalloc
    fn.argtypes = [ctypes.POINTER(q4.q4_matrix), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def test_noalloc_matches_workspace_entry_point_and_oracle():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    fn = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for n, k in SHAPES:
        seed, wstream = 41, n + 7 * k
        w = synth.matrix(seed, wstream, n, k, synth.WEIGHT_STD, device="cuda")
        m = q4.pack(w)
        del w
        x = synth.normal(seed, wstream + 1, 0, k, 1.0).numpy()
        xg = torch.from_numpy(x).cuda()
        y_ws = q4.gemv(m, xg)                       # existing entry point, caller workspace
        rows = sample_rows(n, 16, n + k)
        y_ref, s = oracle_rows(seed, wstream, k, rows, x)
        cm = m.c()
        for call in range(2):
            y = torch.full((n,), float("nan"), device="cuda")
            status = fn(ctypes.byref(cm), xg.data_ptr(), y.data_ptr(), stream)
            assert status == 0, q4.status_string(status)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int32), y_ws.view(torch.int32)), \
                f"{n}x{k} call {call}: differs from q4_gemv"
            assert_gemv_close(y.cpu().numpy()[rows][None, :], y_ref[None, :], s[None, :],
                              f"{n}x{k} noalloc call {call}")
    assert q4.noalloc_status() == 0


def test_noalloc_rejects_matrices_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    fn = _noalloc()
    n, k = 65536, 57344   # K in 4 splits: tickets and partial sums of 1.3 MB, beyond 1 MiB
    assert q4.workspace_bytes(n, k, 1) > (1 << 20)
    m = q4.q4_matrix(256, 256, n, k)  # never dereferenced: rejected before any launch
    assert fn(ctypes.byref(m), 256, 256, None) == 3
    assert np.isfinite(q4.noalloc_status())
