"""The C-ABI library on the CPU: it loads, exports what include/*.h declares,
rejects bad arguments before touching CUDA, and its launch plans replay cleanly."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

import oracle
from quantized_decode_q4_b200 import q4, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(q4_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "q4_gemv" in names and "q4_layer_stack" in names and len(names) >= 20
    lib = ctypes.CDLL(q4.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    assert q4.status_string(0) == "ok"
    assert "misaligned" in q4.status_string(2)
    assert q4.status_string(99) == "unknown status"


def test_argument_errors_before_cuda():
    L = q4.lib()
    m = q4.q4_matrix(16, 16, 4, 33)  # k not a multiple of 32
    assert L.q4_gemv(ctypes.byref(m), 16, 16, 256, 1 << 20, None) == 1
    m = q4.q4_matrix(16, 16, 0, 64)  # n < 1
    assert L.q4_gemv(ctypes.byref(m), 16, 16, 256, 1 << 20, None) == 1
    m = q4.q4_matrix(24, 16, 4, 64)  # qs not 16-byte aligned
    assert L.q4_gemv(ctypes.byref(m), 16, 16, 256, 1 << 20, None) == 2
    m = q4.q4_matrix(16, 16, 4, 64)
    assert L.q4_gemv(ctypes.byref(m), 20, 16, 256, 1 << 20, None) == 2   # x misaligned
    assert L.q4_gemv(ctypes.byref(m), 16, 16, 0, 1 << 20, None) == 3     # no workspace
    assert L.q4_gemv(ctypes.byref(m), 16, 16, 256, 8, None) == 3         # too small
    assert L.q4_gemv(ctypes.byref(m), 16, 16, 272, 1 << 20, None) == 2   # ws alignment
    assert L.q4_gemv_batched(ctypes.byref(m), 16, 0, 16, 256, 1 << 20, None) == 4
    assert L.q4_gemv_batched(ctypes.byref(m), 16, 17, 16, 256, 1 << 20, None) == 4
    assert L.q4_gemv(None, 16, 16, 256, 1 << 20, None) == 1
    assert L.q4_pack(16, ctypes.byref(q4.q4_matrix(16, 16, 4, 40)), None) == 1
    assert L.q4_dequant(ctypes.byref(m), 8, None) == 2


def test_stack_group_rules():
    L = q4.lib()
    mats = (q4.q4_matrix * 3)(*[q4.q4_matrix(256, 256, 64, 64)] * 3)
    xs = (ctypes.c_void_p * 3)(512, 512, 512)
    ys = (ctypes.c_void_p * 3)(1024, 1024, 1024)
    bad = (ctypes.c_int * 3)(0, 2, 1)   # groups must not decrease
    s = q4.q4_stack(3, mats, xs, ys, bad)
    assert L.q4_layer_stack(ctypes.byref(s), 1, 256, 1 << 20, None) == 1
    assert L.q4_stack_workspace_bytes(ctypes.byref(s), 1) == 0
    ok = (ctypes.c_int * 3)(0, 0, 1)
    s = q4.q4_stack(3, mats, xs, ys, ok)
    assert L.q4_stack_workspace_bytes(ctypes.byref(s), 1) >= 256
    nine = (q4.q4_matrix * 9)(*[q4.q4_matrix(256, 256, 64, 64)] * 9)
    x9 = (ctypes.c_void_p * 9)(*[512] * 9)
    g9 = (ctypes.c_int * 9)(*[0] * 9)   # more than 8 GEMVs in a group
    s = q4.q4_stack(9, nine, x9, x9, g9)
    assert L.q4_stack_workspace_bytes(ctypes.byref(s), 1) == 0


def _all_shapes():
    shapes = set()
    for wl in synth.workloads().values():
        for g in wl.gemvs:
            shapes.add((g.n, g.k))
    return sorted(shapes)


EDGE_SHAPES = [(1, 32), (17, 32), (1, 96), (5, 64), (33, 4128), (3, 28672), (50257, 768),
               (16, 4096), (15, 4096), (2, 131072)]


def _groups_of_workloads():
    out = set()
    for wl in synth.workloads().values():
        groups = {}
        for g in wl.gemvs:
            groups.setdefault(g.group, []).append((g.n, g.k))
        out |= {tuple(v) for v in groups.values()}
    return sorted(out)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("num_sms", [148, 132, 160, 7])
def test_batch1_plans_replay_on_host(num_sms, b):
    """Every byte the batch-1 kernel reads was copied from the right place and its
    lane reads the scale of its own block, every (row, slice) is covered once, the
    shared-memory layout fits two CTAs per SM, split-K scratch stays inside the
    workspace - for every workload shape and group, the edge shapes, and devices
    with other multiprocessor counts."""
    for s in _all_shapes() + EDGE_SHAPES + [(1000, 2080), (3, 992), (4096, 14368)]:
        assert q4.check_b1([s], num_sms, b) == 0, (s, num_sms, b)
    for shapes in _groups_of_workloads():
        assert q4.check_b1(list(shapes), num_sms, b) == 0, (shapes, num_sms, b)
    assert q4.check_b1([(5, 96), (700, 2080), (3, 4160)], num_sms, b) == 0
    assert q4.check_b1([(8, 65536)] * 8, num_sms, b) == 0


def test_batch1_plans_replay_random_groups():
    """Seeded random groups of 1..8 GEMVs (tiny to 32768-wide K, ragged rows and
    slices), including narrow groups whose K is split across CTAs."""
    rng = np.random.default_rng(2024)
    ns = [1, 2, 3, 5, 17, 31, 64, 100, 128, 147, 148, 149, 300, 1000, 2368, 4096, 5000]
    kbs = [1, 2, 3, 7, 16, 31, 32, 33, 64, 100, 127, 128, 129, 200, 256, 448, 449, 1000]
    for _ in range(200):
        shapes = [(int(rng.choice(ns)), 32 * int(rng.choice(kbs)))
                  for _ in range(int(rng.integers(1, 9)))]
        assert q4.check_b1(shapes, 148, 1 + len(shapes) % 4) == 0, shapes
    rng = np.random.default_rng(7)
    for _ in range(40):
        shapes = [(int(rng.integers(1, 9)), 32 * int(rng.choice([1024, 1500, 2048, 4096])))
                  for _ in range(int(rng.integers(3, 9)))]
        assert q4.check_b1(shapes) == 0, shapes


def test_batch1_plan_properties():
    gate_up = q4.plan_info([(14336, 4096), (14336, 4096)])
    # K of 4 slices in one piece: no split, one piece per multiprocessor (the
    # second CTA slot of each SM is left to the next launch)
    assert gate_up["splits"] == [1, 1] and gate_up["pieces"] == 148
    assert gate_up["ws_bytes"] == 256
    assert gate_up["smem"] <= 113 * 1024          # two CTAs share an SM
    assert gate_up["slots"] >= 16                  # a deep weight ring
    down = q4.plan_info([(4096, 14336)])
    # 14 slices in splits of at most 4: tickets (one word per row reserved) and
    # partial sums [splits][n]
    assert down["splits"] == [4] and down["slots"] >= 16 and 144 <= down["pieces"] <= 148
    assert down["ws_bytes"] == 256 + 4096 * 4 + 4 * 4096 * 4
    single = q4.plan_info([(768, 768)])           # K within one slice: no split
    assert single["splits"] == [1] and single["ws_bytes"] == 256
    narrow = q4.plan_info([(2, 131072)])
    assert narrow["splits"] == [128] and narrow["pieces"] == 128


def test_register_unpack_on_host():
    assert q4.check_unpack(12345, 500000) == 0


def _check_tc(shapes, b):
    L = q4.lib()
    f = L.q4_debug_check_tc
    f.argtypes = [ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64), ctypes.c_int,
                  ctypes.c_int]
    f.restype = ctypes.c_int
    n = (ctypes.c_int64 * len(shapes))(*[s[0] for s in shapes])
    k = (ctypes.c_int64 * len(shapes))(*[s[1] for s in shapes])
    return f(n, k, len(shapes), b)


def test_tensor_core_plans_replay_on_host():
    """Every (tile, block) of the batched kernel is covered once, every TMA box
    and operand row is in bounds, every split tile's pieces take slots 0..p-1."""
    extra = [(127, 32), (129, 64), (128, 8192), (2048, 256), (1000, 2080), (5, 14336),
             (128256, 4096)]
    for s in _all_shapes() + EDGE_SHAPES + extra:
        for b in (2, 3, 8, 9, 16):
            assert _check_tc([s], b) == 0, (s, b)
    for wl in synth.workloads().values():
        groups = {}
        for g in wl.gemvs:
            groups.setdefault(g.group, []).append((g.n, g.k))
        for shapes in {tuple(v) for v in groups.values()}:
            for b in (2, 16):
                assert _check_tc(list(shapes), b) == 0, (shapes, b)
    assert _check_tc([(5, 96), (700, 2080), (3, 4160)], 4) == 0
    assert _check_tc([(5, 96)], 1) != 0 and _check_tc([(5, 96)], 17) != 0


def test_tensor_core_plans_replay_random_groups():
    """Seeded random groups of 1..8 GEMVs (ragged 128-row tiles, block counts that are
    and are not multiples of the 8-block window) for every token count 2..16."""
    rng = np.random.default_rng(99)
    ns = [1, 7, 127, 128, 129, 300, 1000, 4096, 5000]
    kbs = [1, 3, 7, 8, 9, 18, 30, 44, 64, 100, 128, 129, 448]
    for _ in range(60):
        shapes = [(int(rng.choice(ns)), 32 * int(rng.choice(kbs)))
                  for _ in range(int(rng.integers(1, 9)))]
        b = int(rng.integers(2, 17))
        assert _check_tc(shapes, b) == 0, (shapes, b)


def test_tensor_core_operands_on_host():
    """The dequantised A operand is q - 8 exactly at every MMA position and an
    emulated MMA over the staged hi/lo activations gives the block sum."""
    L = q4.lib()
    f = L.q4_debug_check_tc_operands
    f.argtypes = [ctypes.c_uint64, ctypes.c_int64]
    f.restype = ctypes.c_int64
    assert f(77, 100000) == 0


def test_integer_block_dot_on_host():
    """Activation digits split exactly; unflagged block sums within 2^-14 of each
    element, flagged blocks (outliers, subnormal neighbours, extreme ranges) on
    the binary32 path within its rounding."""
    L = q4.lib()
    f = L.q4_debug_check_intdot
    f.argtypes = [ctypes.c_uint64, ctypes.c_int64]
    f.restype = ctypes.c_int64
    assert f(2024, 300000) == 0


def test_interchange_matches_oracle():
    rng = np.random.default_rng(5)
    n, k = 7, 96
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    blocks = oracle.q4_pack(w)
    qs_o, d_o = oracle.blocks_to_planes(blocks, n, k)
    qs, d = q4.blocks_to_planes(blocks, n, k)
    assert np.array_equal(qs, qs_o) and np.array_equal(d, d_o)
    assert np.array_equal(q4.planes_to_blocks(qs, d, n, k), blocks)
