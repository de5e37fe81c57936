"""The oracle against what the block definition, the mathematics and numpy fix."""
import numpy as np
import pytest

import pins


def test_fp16_conversions_match_ieee(oracle_lib):
    pins.check_fp16(oracle_lib)


def test_golden_hand_cases(oracle_lib):
    pins.check_golden(oracle_lib)


def test_dequant_exact_for_every_scale_and_code(oracle_lib):
    pins.check_dequant_exact(oracle_lib)


def test_roundtrip_bound_million_blocks(oracle_lib):
    stats = pins.check_roundtrip(oracle_lib, 1_000_000)
    # clamping happens (the side opposite m) but rarely
    assert 0 < stats["clamped_fraction"] < 0.01


def test_gemv_matches_exact_rational_sum(oracle_lib):
    pins.check_gemv_exact(oracle_lib)


def test_rejects_k_not_multiple_of_32(oracle_lib):
    import ctypes

    import oracle
    with pytest.raises(ValueError):
        oracle.q4_pack(np.zeros((1, 33), np.float32))
    w = np.zeros(33, np.float32)
    out = np.zeros(36, np.uint8)
    rc = oracle_lib.oracle_q4_pack(oracle._ptr(w, ctypes.c_float), 1, 33,
                                   oracle._ptr(out, ctypes.c_uint8))
    assert rc == -1 and not out.any()


def test_linearity_and_one_hot(oracle_lib):
    import oracle
    rng = np.random.default_rng(3)
    n, k = 5, 96
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    blocks = oracle.q4_pack(w)
    w_hat = oracle.q4_dequant(blocks, n, k)
    for kk in (0, 17, 31, 32, 95):
        x = np.zeros(k, np.float32)
        x[kk] = 1.0
        y, _ = oracle.q4_gemv(blocks, n, k, x)
        assert np.array_equal(y, w_hat[:, kk].astype(np.float64))
    x1 = rng.standard_normal(k).astype(np.float32)
    y1, _ = oracle.q4_gemv(blocks, n, k, x1)
    y2, _ = oracle.q4_gemv(blocks, n, k, (2 * x1).astype(np.float32))
    assert np.array_equal(y2, 2 * y1)  # scaling by 2 is exact in binary floating point
