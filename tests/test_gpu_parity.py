"""GPU parity: the CUDA library against the oracle, element by element.

pack and dequant must be bit-exact; GEMV outputs must satisfy
|y - y_ref| <= 1e-4 * sum|w_hat x| + 1e-6 per element (y_ref in binary64).
Small cases compare every output; the full-size decode steps compare sampled rows,
whose binary32 weights the host re-draws independently of the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (assert_gemv_close, gpu_matrix_from_host, oracle_planes, oracle_rows,
                         planes_to_host, sample_rows)
from quantized_decode_q4_b200 import q4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    torch.cuda.init()


def host_matrix(seed, stream, n, k, std=synth.WEIGHT_STD):
    return synth.matrix(seed, stream, n, k, std).numpy()


# ---------------------------------------------------------------------------
# generator on the GPU
# ---------------------------------------------------------------------------

def test_generator_on_gpu_matches_host():
    a = synth.normal(4, 77, 123456, 300000, 0.02, device="cuda").cpu().numpy()
    b = synth.normal_np(4, 77, 123456, 300000, 0.02)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# ---------------------------------------------------------------------------
# pack and dequant: bit-exact
# ---------------------------------------------------------------------------

PACK_SHAPES = [(1, 32), (3, 96), (17, 768), (64, 4096), (5, 14336), (130, 960), (7, 1408),
               (33, 4128), (40, 576)]


@pytest.mark.parametrize("shape", PACK_SHAPES)
def test_pack_and_dequant_bit_exact(shape):
    n, k = shape
    w = host_matrix(9, n * 7 + k, n, k)
    blocks, qs_o, d_o = oracle_planes(w)
    m = gpu_matrix_from_host(w)
    qs, d = planes_to_host(m)
    assert np.array_equal(qs, qs_o), "code bytes differ"
    assert np.array_equal(d, d_o), "scale bits differ"
    w_hat = q4.dequant(m).cpu().numpy()
    assert np.array_equal(w_hat.view(np.uint32), oracle.q4_dequant(blocks, n, k).view(np.uint32))


def special_rows():
    import pins
    rows = []
    for case in pins.golden_cases():
        if case["name"][0] == "H6":
            rows.extend(pins.h6_weights().reshape(-1, 32))
        else:
            rows.append(np.array(case["w"], np.float32))
    rng = np.random.default_rng(1)
    rows.append(np.full(32, -0.0, np.float32))                       # negative zeros
    rows.append((rng.standard_normal(32) * 1e-5).astype(np.float32))  # subnormal binary16 d
    rows.append((rng.standard_normal(32) * 3e4).astype(np.float32))   # large scale
    t = rng.standard_normal(32).astype(np.float32)
    t[9] = -np.abs(t).max()
    t[20] = -t[9]                                                     # tie, opposite signs
    rows.append(t)
    rows.append(np.linspace(-1, 1, 32, dtype=np.float32))
    rows.extend(pins.roundtrip_blocks(4000, seed=3))
    return np.stack(rows).astype(np.float32)


def test_pack_special_blocks_bit_exact():
    r = special_rows()
    w = r.reshape(-1, 64) if r.shape[0] % 2 == 0 else r[:-1].reshape(-1, 64)
    n, k = w.shape
    blocks, qs_o, d_o = oracle_planes(w)
    m = gpu_matrix_from_host(w)
    qs, d = planes_to_host(m)
    assert np.array_equal(qs, qs_o) and np.array_equal(d, d_o)
    w_hat = q4.dequant(m).cpu().numpy()
    assert np.array_equal(w_hat.view(np.uint32), oracle.q4_dequant(blocks, n, k).view(np.uint32))


# ---------------------------------------------------------------------------
# GEMV, batch 1 and small batches: every output
# ---------------------------------------------------------------------------

def _all_workload_shapes():
    s = set()
    for wl in synth.workloads().values():
        for g in wl.gemvs:
            s.add((g.n, g.k))
    return sorted(s)


EDGE_SHAPES = [(1, 32), (17, 32), (1, 96), (5, 64), (16, 4096), (15, 4128), (33, 4128),
               (3, 28672), (2, 131072), (100, 14336)]
FULL_CHECK_LIMIT = 3_000_000   # weights drawn on the host for a full comparison


def _run_full(n, k, b, seed=21):
    w = host_matrix(seed, n + 3 * k + b, n, k)
    X = synth.normal(seed, 1000 + n + k, 0, b * k, 1.0).numpy().reshape(b, k)
    blocks = oracle.q4_pack(w)
    Y_ref, S = oracle.q4_gemv_batched(blocks, n, k, X)
    m = gpu_matrix_from_host(w)
    Xg = torch.from_numpy(X).cuda()
    if b == 1:
        y = q4.gemv(m, Xg[0]).cpu().numpy()[None, :]
    else:
        y = q4.gemv_batched(m, Xg).cpu().numpy()
    return assert_gemv_close(y, Y_ref, S, f"{n}x{k} b={b}")


@pytest.mark.parametrize("shape", [s for s in _all_workload_shapes() + EDGE_SHAPES
                                   if s[0] * s[1] <= FULL_CHECK_LIMIT])
def test_gemv_b1_every_output(shape):
    _run_full(*shape, b=1)


@pytest.mark.parametrize("b", [2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("shape", [(1, 32), (17, 768), (192, 576), (130, 1408), (64, 4096),
                                   (33, 4128)])
def test_gemv_batched_every_output(shape, b):
    _run_full(*shape, b=b)


@pytest.mark.parametrize("b", [5, 6, 9, 12, 16])
@pytest.mark.parametrize("shape", [(127, 32), (129, 64), (128, 8192), (2048, 256), (300, 960),
                                   (1000, 2080), (5, 14336)])
def test_gemv_tensor_core_every_output(shape, b):
    """Ragged last tiles, one-block rows, tiles split over many CTAs, every
    compiled token width (2, 4, 8, 16) with absent tokens."""
    _run_full(*shape, b=b)


@pytest.mark.parametrize("shape", [s for s in _all_workload_shapes()
                                   if s[0] * s[1] > FULL_CHECK_LIMIT])
@pytest.mark.parametrize("b", [1, 4, 16])
def test_gemv_full_size_sampled_rows(shape, b):
    n, k = shape
    seed, stream = 31, 2 * (n + k)
    wg = synth.matrix(seed, stream, n, k, synth.WEIGHT_STD, device="cuda")
    m = q4.pack(wg)
    rows = sample_rows(n, 24, n + k)
    # the GPU drew the same binary32 weights as the host does for these rows
    w_rows = synth.matrix_rows(seed, stream, k, rows, synth.WEIGHT_STD).numpy()
    assert np.array_equal(wg[rows].cpu().numpy(), w_rows)
    del wg
    X = synth.normal(seed, stream + 1, 0, b * k, 1.0).numpy().reshape(b, k)
    Xg = torch.from_numpy(X).cuda()
    y = (q4.gemv(m, Xg[0])[None, :] if b == 1 else q4.gemv_batched(m, Xg)).cpu().numpy()
    Y_ref, S = oracle_rows(seed, stream, k, rows, X)
    assert_gemv_close(y[:, rows], Y_ref, S, f"{n}x{k} b={b}")


def test_zero_matrix_gives_exact_zero():
    w = np.zeros((40, 960), np.float32)
    m = gpu_matrix_from_host(w)
    x = torch.randn(960, device="cuda")
    assert torch.count_nonzero(q4.gemv(m, x)).item() == 0


def test_deterministic_and_workspace_reusable():
    n, k = 1024, 4096   # split-K path
    wg = synth.matrix(5, 5, n, k, synth.WEIGHT_STD, device="cuda")
    m = q4.pack(wg)
    x = synth.normal(5, 6, 0, k, 1.0, device="cuda")
    ws = q4.workspace(q4.workspace_bytes(n, k, 4))
    ys = [q4.gemv(m, x, ws=ws).clone() for _ in range(5)]
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int32), ys[0].view(torch.int32))
    X = synth.normal(5, 7, 0, 4 * k, 1.0, device="cuda").view(4, k)
    Y1 = q4.gemv_batched(m, X, ws=ws).clone()
    Y2 = q4.gemv_batched(m, X, ws=ws).clone()
    assert torch.equal(Y1, Y2)
    torch.cuda.synchronize()
    assert q4.workspace_status(ws) == 0
    # tickets were reset: the workspace past the header is all zero again
    assert torch.count_nonzero(ws[256:256 + 4 * 64]).item() == 0


def test_launch_counter_counts_kernels():
    m = gpu_matrix_from_host(host_matrix(3, 3, 64, 256))
    x = torch.randn(256, device="cuda")
    c0 = q4.launch_count()
    q4.gemv(m, x)
    q4.gemv_batched(m, torch.randn(6, 256, device="cuda"))  # one tensor-core launch
    assert q4.launch_count() - c0 == 2


def test_workspace_shared_by_different_shapes():
    """Calls with different split-K layouts reuse one workspace in any order."""
    shapes = [(1024, 4096), (128, 512), (4096, 14336), (1408, 512), (1024, 4096)]
    need = max(q4.workspace_bytes(n, k, 4) for n, k in shapes)
    ws = q4.workspace(need)
    for i, (n, k) in enumerate(shapes):
        w = host_matrix(13, i, n, k) if n * k <= FULL_CHECK_LIMIT else None
        if w is None:
            wg = synth.matrix(13, i, n, k, synth.WEIGHT_STD, device="cuda")
            m = q4.pack(wg)
            rows = sample_rows(n, 16, i)
            w_rows = synth.matrix_rows(13, i, k, rows, synth.WEIGHT_STD).numpy()
        else:
            m = gpu_matrix_from_host(w)
            rows = list(range(n))
            w_rows = w
        for b in (1, 3):
            X = synth.normal(13, 500 + i, 0, b * k, 1.0).numpy().reshape(b, k)
            Y = q4.gemv_batched(m, torch.from_numpy(X).cuda(), ws=ws).cpu().numpy()
            Y_ref, S = oracle.q4_gemv_batched(oracle.q4_pack(w_rows), len(rows), k, X)
            assert_gemv_close(Y[:, rows], Y_ref, S, f"{n}x{k} b={b} shared ws")
