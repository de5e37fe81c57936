"""Helpers for the GPU-vs-oracle parity tests.

Inputs come from the shared seeded generator (quantized_decode_q4_b200.synth) only;
expected values come from the oracle only. Both sides draw the same binary32
numbers: either on the host for the oracle and uploaded for the GPU, or on the GPU
and re-drawn on the host for the rows the oracle checks.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_decode_q4_b200 import q4, synth

REL_TOL = 1e-4
ABS_TOL = 1e-6


def oracle_planes(w: np.ndarray):
    n, k = w.shape
    blocks = oracle.q4_pack(w)
    qs, d = oracle.blocks_to_planes(blocks, n, k)
    return blocks, qs, d


def assert_gemv_close(y_gpu, y_ref, abs_sum, what=""):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = REL_TOL * abs_sum + ABS_TOL
    bad = np.flatnonzero(~(err <= bound))
    assert bad.size == 0, (f"{what}: {bad.size} of {y_ref.size} outputs outside tolerance; "
                           f"first flat indexes {bad[:5]}: gpu {y_gpu.ravel()[bad[:5]]} "
                           f"ref {y_ref.ravel()[bad[:5]]}")
    return float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0


def gpu_matrix_from_host(w: np.ndarray) -> q4.Q4Matrix:
    wt = torch.from_numpy(np.ascontiguousarray(w)).cuda()
    return q4.pack(wt)


def planes_to_host(m: q4.Q4Matrix):
    qs = m.qs_plane().cpu().numpy()
    d = m.d_plane().cpu().numpy().view(np.uint16)
    return qs, d


def sample_rows(n: int, count: int, seed: int):
    """First, last and `count` random rows (sorted, unique)."""
    rng = np.random.default_rng(seed)
    rows = {0, n - 1} | set(rng.integers(0, n, min(count, n)).tolist())
    return sorted(rows)


def oracle_rows(seed: int, stream: int, k: int, rows, x: np.ndarray):
    """Oracle y (and abs sums) for the listed rows of a synthetic weight matrix."""
    w = synth.matrix_rows(seed, stream, k, rows, synth.WEIGHT_STD).numpy()
    blocks = oracle.q4_pack(w)
    if x.ndim == 1:
        return oracle.q4_gemv(blocks, len(rows), k, x)
    return oracle.q4_gemv_batched(blocks, len(rows), k, x)
