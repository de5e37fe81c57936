"""B200-native Q4_0 decode GEMV: a C-ABI CUDA library (libq4_b200.so) and its binding.

    from quantized_decode_q4_b200 import q4
    m = q4.pack(w)            # binary32 [n][k] on the GPU -> Q4_0 planes
    y = q4.gemv(m, x)         # y = W x, batch 1
"""
from . import _lib as q4  # noqa: F401
