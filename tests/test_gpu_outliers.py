"""Batch-1 GEMV parity for activation blocks with outliers, element by element
against the oracle, within |y - y_ref| <= 1e-4 * sum|w_hat x| + 1e-6.

The batch-1 kernel multiplies most activation blocks in 31-bit block fixed point.
An outlier inflates its block's scale, so its neighbours would round coarsely;
such blocks must take the kernel's exact binary32 path. The outliers sit on
weights whose code is 8 (a zero weight column), so they add nothing to
sum|w_hat x| while they set the block's scale: the case where a fixed-point
error would show most. Inputs are built here from the shared seeded generator;
expected values come from the oracle only.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_gemv_close, gpu_matrix_from_host
from quantized_decode_q4_b200 import q4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _case(n, k, seed, factor, per_block, signs, rest="normal"):
    """W N(0, 0.02) with zero columns at the outlier positions (code 8 in every row);
    x N(0, 1) (or subnormal) with `per_block` outliers of `factor` x the block's
    typical |x| in every block, signs from `signs`."""
    w = synth.matrix(seed, 1, n, k, synth.WEIGHT_STD).numpy().copy()
    x = synth.normal(seed, 2, 0, k, 1.0).numpy().astype(np.float64)
    rng = np.random.default_rng(seed)
    if rest == "subnormal":
        x = x * 1e-40
    cols = []
    for b in range(k // 32):
        pos = rng.choice(32, size=per_block, replace=False)
        typical = np.median(np.abs(x[32 * b: 32 * b + 32])) or 1.0
        for i, p in enumerate(pos):
            c = 32 * b + int(p)
            x[c] = signs[i % len(signs)] * factor * (typical if rest == "normal" else 1.0)
            cols.append(c)
    w[:, cols] = 0.0
    return w.astype(np.float32), x.astype(np.float32)


def _check(w, x, what):
    n, k = w.shape
    blocks = oracle.q4_pack(w)
    y_ref, s = oracle.q4_gemv(blocks, n, k, x)
    m = gpu_matrix_from_host(w)
    y = q4.gemv(m, torch.from_numpy(x).cuda()).cpu().numpy()
    assert_gemv_close(y[None, :], y_ref[None, :], s[None, :], what)


@pytest.mark.parametrize("factor", [1e3, 1e4, 1e5, 1e6])
@pytest.mark.parametrize("per_block,signs", [(1, [1.0]), (2, [1.0, -1.0]), (2, [-1.0, -1.0])])
@pytest.mark.parametrize("shape", [(64, 4096), (33, 4128), (300, 960)])
def test_outliers_on_code_8(shape, factor, per_block, signs):
    n, k = shape
    w, x = _case(n, k, 17 + n, factor, per_block, signs)
    _check(w, x, f"{n}x{k} outliers {per_block} x {factor:g}")


@pytest.mark.parametrize("shape", [(64, 4096), (40, 576)])
def test_subnormal_neighbours(shape):
    """Each block: one element of 1.0 (code 8) and the rest subnormal."""
    n, k = shape
    w, x = _case(n, k, 5, 1.0, 1, [1.0], rest="subnormal")
    assert np.count_nonzero((np.abs(x) < 1.2e-38) & (x != 0)) > k // 2
    _check(w, x, f"{n}x{k} subnormal neighbours")


def test_outliers_in_some_blocks_only():
    """Outliers in a few blocks of a wide matrix: those slices take the exact
    path, the others stay on the integer path, every output still within tolerance."""
    n, k = 256, 14336
    w = synth.matrix(8, 1, n, k, synth.WEIGHT_STD).numpy().copy()
    x = synth.normal(8, 2, 0, k, 1.0).numpy().copy()
    for c in (5, 1030, 7000, 14335):
        x[c] = 3e5 * (1 if c % 2 else -1)
        w[:, c] = 0.0
    _check(w, x, "256x14336 sparse outliers")


def test_wide_dynamic_range_without_outlier_weights():
    """Activations spanning 2^-20 .. 2^20 inside every block, ordinary weights."""
    n, k = 128, 4096
    w = synth.matrix(9, 1, n, k, synth.WEIGHT_STD).numpy()
    u = synth.normal(9, 2, 0, k, 1.0).numpy()
    e = (np.arange(k) % 41 - 20).astype(np.float32)
    x = (u * np.exp2(e)).astype(np.float32)
    _check(w, x, "128x4096 wide range")
