"""Pins for the oracle: checks against values that do not come from the oracle's code.

Each check takes a loaded oracle library (so that the planted-mistake test can run
the same checks on deliberately broken copies) and raises AssertionError when the
library disagrees with what the block definition, the mathematics or an
independent library routine fixes.

  * fp16: numpy's binary16 conversion (IEEE round to nearest even) on every
    binary16 pattern, every halfway point and random binary32 patterns.
  * golden: hand-derived blocks in tests/golden/ (each with its derivation).
  * dequant: w_hat = d * (q - 8) evaluated exactly in binary64 for every finite
    binary16 d and all 16 codes.
  * round trip: |w - w_hat| <= |d|/2 + 8 |d - d_h| + 2^-18 |d| for unclamped
    weights (|d| + ... for the clamped side), over 10^6 random blocks.
  * gemv: exact rational arithmetic (fractions.Fraction) on tiny matrices, the
    oracle's binary64 sum within the recursive-summation bound.
"""
from __future__ import annotations

import glob
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
BLOCK_DTYPE = np.dtype([("d", "<u2"), ("qs", "u1", (16,))])


# ----------------------------------------------------------------------------
# fixtures
# ----------------------------------------------------------------------------

def load_golden(path: str) -> dict:
    out = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.split()
    return out


def golden_cases() -> list:
    return [load_golden(p) for p in sorted(glob.glob(os.path.join(GOLDEN_DIR, "h*.txt")))]


def h6_weights() -> np.ndarray:
    """The H6 construction rule, expanded (see tests/golden/h6_rule.txt)."""
    n, k = 2, 128
    w = np.zeros((n, k), dtype=np.float32)
    for r in range(n):
        for b in range(4):
            s = (b + 1 + 4 * r) / 8.0
            for j in range(32):
                c = 0 if j == 0 else (5 * j + 3 * b + r) % 16
                w[r, 32 * b + j] = s * (c - 8)
    return w


def decode_blocks_exact(blocks: np.ndarray, n: int, k: int):
    """Independent decode of llama.cpp-layout blocks to exact rationals (no oracle code)."""
    raw = np.ascontiguousarray(blocks, dtype=np.uint8).reshape(-1)
    view = raw.view(BLOCK_DTYPE).reshape(n, k // 32)
    d = view["d"].view(np.float16).astype(np.float64)
    qs = view["qs"]
    lo = (qs & 0x0F).astype(np.int64)
    hi = (qs >> 4).astype(np.int64)
    codes = np.concatenate([lo, hi], axis=-1)  # [n, nb, 32]: j<16 low nibbles, j>=16 high
    w = [[Fraction(float(d[r, b])) * int(codes[r, b, j] - 8)
          for b in range(k // 32) for j in range(32)] for r in range(n)]
    return w


# ----------------------------------------------------------------------------
# checks
# ----------------------------------------------------------------------------

def check_fp16(lib) -> None:
    """binary16 conversions against numpy on every pattern, every tie and random inputs."""
    allh = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref32 = allh.view(np.float16).astype(np.float32)
    got32 = np.array([lib.oracle_f16_to_f32(int(h)) for h in allh], dtype=np.float32)
    nan = np.isnan(ref32)
    assert np.array_equal(np.isnan(got32), nan), "NaN patterns must decode to NaN"
    assert np.array_equal(got32[~nan].view(np.uint32), ref32[~nan].view(np.uint32)), \
        "f16->f32 differs from numpy"
    back = np.array([lib.oracle_f32_to_f16(float(v)) for v in got32[~nan]], dtype=np.uint16)
    assert np.array_equal(back, allh[~nan]), "f16->f32->f16 must round-trip"
    for v in got32[nan][:64]:
        h = lib.oracle_f32_to_f16(float(v))
        assert (h & 0x7C00) == 0x7C00 and (h & 0x3FF) != 0, "NaN must stay NaN"
    # halfway points between consecutive finite halves (exact in binary32): ties to even
    fin = allh[np.isfinite(ref32)].astype(np.int64)
    pos = fin[(fin < 0x7BFF)]
    a = pos.astype(np.uint16).view(np.float16).astype(np.float64)
    b = (pos + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = ((a + b) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (a + b) / 2)
    mids = np.concatenate([mid, -mid])
    rng = np.random.default_rng(12345)
    rnd = rng.integers(0, 1 << 32, 200000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    specials = np.array([0.25, -0.25, 65504.0, 65519.996, 65520.0, 1e6, -1e6, 2.0 ** -24,
                         2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 6e-8, 0.0, -0.0,
                         np.float32(1e-40)], dtype=np.float32)
    vals = np.concatenate([mids, rnd, specials]).astype(np.float32)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([lib.oracle_f32_to_f16(float(v)) for v in vals], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"f32->f16 differs from numpy at {vals[bad[:5]]}"
    assert lib.oracle_f32_to_f16(0.25) == 0x3400 and lib.oracle_f32_to_f16(-0.25) == 0xB400


def check_golden(lib) -> None:
    """Hand-derived blocks: pack bytes, dequant, y and abs_sum."""
    for case in golden_cases():
        n, k = int(case["n"][0]), int(case["k"][0])
        if case["name"][0] == "H6":
            w = h6_weights()
        else:
            w = np.array(case["w"], dtype=np.float32).reshape(n, k)
        blocks = oracle.q4_pack(w, lib=lib)
        view = blocks.reshape(-1).view(BLOCK_DTYPE)
        want_d = np.array([int(h, 16) for h in case["d_bits"]], dtype=np.uint16)
        assert np.array_equal(view["d"], want_d), f"{case['name']}: d bits {view['d']}"
        w_hat = oracle.q4_dequant(blocks, n, k, lib=lib)
        if case["name"][0] == "H6":
            assert np.array_equal(w_hat, w), "H6: packing must be exact"
            for kk in range(k):
                x = np.zeros(k, dtype=np.float32)
                x[kk] = 1.0
                y, s = oracle.q4_gemv(blocks, n, k, x, lib=lib)
                assert np.array_equal(y, w[:, kk].astype(np.float64)), f"H6 column {kk}"
                assert np.array_equal(s, np.abs(w[:, kk]).astype(np.float64))
            qs_plane, d_plane = oracle.blocks_to_planes(blocks, n, k, lib=lib)
            assert np.array_equal(d_plane.reshape(-1), want_d)
            assert np.array_equal(qs_plane.reshape(-1), view["qs"].reshape(-1))
            continue
        want_qs = bytes.fromhex("".join(case["qs"]))
        assert view["qs"].tobytes() == want_qs, f"{case['name']}: qs {view['qs'].tobytes().hex()}"
        want_w = np.array(case["w_hat"], dtype=np.float32).reshape(n, k)
        assert np.array_equal(w_hat, want_w), f"{case['name']}: w_hat"
        x = np.array(case["x"], dtype=np.float32)
        y, s = oracle.q4_gemv(blocks, n, k, x, lib=lib)
        assert y[0] == float(case["y"][0]), f"{case['name']}: y={y}"
        assert s[0] == float(case["abs_sum"][0]), f"{case['name']}: abs_sum={s}"
        qs_plane, d_plane = oracle.blocks_to_planes(blocks, n, k, lib=lib)
        assert qs_plane.tobytes() == want_qs and np.array_equal(d_plane.reshape(-1), want_d)


def check_dequant_exact(lib) -> None:
    """Every finite binary16 d times every code: w_hat equals d*(q-8) computed exactly."""
    allh = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = np.isfinite(allh.view(np.float16))
    ds = allh[finite]
    nblk = ds.size
    blocks = np.zeros(nblk, dtype=BLOCK_DTYPE)
    blocks["d"] = ds
    # codes 0..15 in the low nibbles (weights 0..15), 15..0 in the high ones (16..31)
    lo = np.arange(16, dtype=np.uint8)
    blocks["qs"] = (lo | ((15 - lo) << 4))[None, :]
    raw = blocks.view(np.uint8).reshape(nblk, 1, 18)
    w_hat = oracle.q4_dequant(raw, nblk, 32, lib=lib)
    codes = np.concatenate([np.arange(16), 15 - np.arange(16)]).astype(np.float64)
    exact = ds.view(np.float16).astype(np.float64)[:, None] * (codes[None, :] - 8.0)
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact), \
        "d*(q-8) must be exact in binary32"
    assert np.array_equal(w_hat.astype(np.float64), exact), "dequant is not d*(q-8)"
    # q = 8 decodes to +/-0 for every d
    assert np.all(w_hat[:, 8] == 0.0) and np.all(w_hat[:, 23] == 0.0)


def roundtrip_blocks(nblocks: int, seed: int = 7) -> np.ndarray:
    """Random blocks over several magnitudes, including binary16-subnormal scales and ties."""
    rng = np.random.default_rng(seed)
    per = nblocks // 4
    parts = [
        rng.standard_normal((per, 32)).astype(np.float32) * np.float32(0.02),
        rng.standard_normal((per, 32)).astype(np.float32),
        rng.standard_normal((per, 32)).astype(np.float32) * np.float32(1e-4),
        rng.standard_t(3, (nblocks - 3 * per, 32)).astype(np.float32),
    ]
    w = np.concatenate(parts)
    # equal-magnitude pairs of opposite sign in some blocks (first index decides)
    idx = rng.integers(0, w.shape[0], w.shape[0] // 50)
    w[idx, 5] = -w[idx, 3]
    w[idx, 3] = np.abs(w[idx]).max(axis=1)
    w[idx, 5] = -w[idx, 3]
    return w


def check_roundtrip(lib, nblocks: int = 1_000_000) -> dict:
    """|w - w_hat| within the rounding bound; clamps only on the side opposite m."""
    w = roundtrip_blocks(nblocks)
    blocks = oracle.q4_pack(w.reshape(-1, 32), lib=lib)  # one block per row
    w_hat = oracle.q4_dequant(blocks, w.shape[0], 32, lib=lib)
    view = blocks.reshape(-1).view(BLOCK_DTYPE)
    d_h = view["d"].view(np.float16).astype(np.float64)
    a = np.abs(w)
    first = np.argmax(a, axis=1)  # numpy argmax returns the first maximum
    m = w[np.arange(w.shape[0]), first]
    d32 = (m / np.float32(-8.0)).astype(np.float64)
    assert np.array_equal(d32.astype(np.float16).astype(np.float64), d_h), "stored d != fp16(m/-8)"
    err = np.abs(w.astype(np.float64) - w_hat.astype(np.float64))
    ad = np.abs(d32)[:, None]
    dd = np.abs(d32 - d_h)[:, None]
    ratio = w.astype(np.float64) / np.where(d32 == 0, 1.0, d32)[:, None]
    clamped = ratio > 7.5 - 2.0 ** -17
    bound = ad * (0.5 + 2.0 ** -18) + 8 * dd
    bound_clamped = ad * (1.0 + 2.0 ** -18) + 8 * dd
    ok = np.where(clamped, err <= bound_clamped, err <= bound)
    assert ok.all(), f"round-trip bound broken in {np.count_nonzero(~ok)} weights"
    # clamped weights have the opposite sign of m (or the ratio would be <= -7.5)
    assert np.all(ratio[clamped] > 0)
    return {"blocks": w.shape[0], "clamped_fraction": float(clamped.mean())}


def check_gemv_exact(lib, cases: int = 40, seed: int = 11) -> None:
    """Tiny random matrices: the binary64 oracle sum is within gamma_{k-1} of the exact sum."""
    rng = np.random.default_rng(seed)
    for c in range(cases):
        n = int(rng.integers(1, 4))
        k = 32 * int(rng.integers(1, 5))
        w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
        x = rng.standard_normal(k).astype(np.float32)
        blocks = oracle.q4_pack(w, lib=lib)
        y, s = oracle.q4_gemv(blocks, n, k, x, lib=lib)
        w_exact = decode_blocks_exact(blocks, n, k)
        # the oracle's binary32 dequant equals the exact rational decode
        w_hat = oracle.q4_dequant(blocks, n, k, lib=lib)
        for r in range(n):
            assert all(Fraction(float(w_hat[r, i])) == w_exact[r][i] for i in range(k))
            terms = [w_exact[r][i] * Fraction(float(x[i])) for i in range(k)]
            exact = sum(terms, Fraction(0))
            sabs = sum((abs(t) for t in terms), Fraction(0))
            tol = (k - 1) * 2.0 ** -53 * float(sabs) * 1.01
            assert abs(float(Fraction(y[r]) - exact)) <= tol, f"case {c} row {r}"
            assert abs(float(Fraction(s[r]) - sabs)) <= tol
        # batched form: token t uses X[t]
        X = rng.standard_normal((3, k)).astype(np.float32)
        Y, S = oracle.q4_gemv_batched(blocks, n, k, X, lib=lib)
        for t in range(3):
            for r in range(n):
                exact = sum((w_exact[r][i] * Fraction(float(X[t, i])) for i in range(k)),
                            Fraction(0))
                sabs = sum((abs(w_exact[r][i] * Fraction(float(X[t, i]))) for i in range(k)),
                           Fraction(0))
                tol = (k - 1) * 2.0 ** -53 * float(sabs) * 1.01
                assert abs(float(Fraction(Y[t, r]) - exact)) <= tol, f"case {c} token {t} row {r}"
                # each token's own sum of |w_hat x| (its tolerance term)
                assert abs(float(Fraction(S[t, r]) - sabs)) <= tol, f"case {c} token {t} row {r}"


ALL_CHECKS = (check_golden, check_dequant_exact, check_gemv_exact, check_fp16)
