"""The bounded-wait timeout path on the GPU without a fault: q4_debug_gemv_stall runs
the real kernels with every stage barrier expecting 16 bytes more than its copies
bring, so every wait runs out (20 ms each); the kernel must return, record
Q4_ERR_TIMEOUT in the workspace, and leave the device usable (tensor memory freed)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_gemv_close, gpu_matrix_from_host
from quantized_decode_q4_b200 import q4, synth

pytestmark = pytest.mark.gpu

Q4_ERR_TIMEOUT = 6


def _stall(m, X, Y, ws):
    f = q4.lib().q4_debug_gemv_stall
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    f.restype = ctypes.c_int
    cm = m.c()
    return f(ctypes.addressof(cm), X.data_ptr(), X.shape[0], Y.data_ptr(), ws.data_ptr(),
             ws.numel(), None)


@pytest.mark.parametrize("b", [1, 2, 16])
def test_waits_run_out_and_device_stays_usable(b):
    # one tile per warp (batch 1) / one stage per CTA (tensor cores)
    n, k = 128, 256
    w = synth.matrix(9, 9, n, k, synth.WEIGHT_STD).numpy()
    m = gpu_matrix_from_host(w)
    X = synth.normal(9, 10, 0, b * k, 1.0).numpy().reshape(b, k)
    Xg = torch.from_numpy(X).cuda()
    Y = torch.empty(b, n, device="cuda")
    ws = q4.workspace(q4.workspace_bytes(n, k, b))
    assert _stall(m, Xg, Y, ws) == 0
    torch.cuda.synchronize()
    assert q4.workspace_status(ws) == Q4_ERR_TIMEOUT
    # the same workspace, cleared, and the same device serve a normal call
    q4.workspace_init(ws)
    Y2 = q4.gemv_batched(m, Xg, ws=ws).cpu().numpy()
    torch.cuda.synchronize()
    assert q4.workspace_status(ws) == 0
    Y_ref, S = oracle.q4_gemv_batched(oracle.q4_pack(w), n, k, X)
    assert_gemv_close(Y2, Y_ref, S, f"after stall b={b}")
