"""Decode steps (layer stacks) on the GPU against the oracle, on sampled rows of
every GEMV; direct launches and graph replays must agree bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_gemv_close, oracle_rows, sample_rows
from quantized_decode_q4_b200 import q4, synth
from quantized_decode_q4_b200.decode_step import DecodeStep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def check_step(step: DecodeStep, rows_per_gemv: int, seed: int):
    wl, b = step.workload, step.batch
    worst = 0.0
    for i, g in enumerate(wl.gemvs):
        X = wl.activations(i, b).numpy()
        assert np.array_equal(step.xs[i].cpu().numpy(), X), "device activations differ"
        rows = sample_rows(g.n, rows_per_gemv, seed + i)
        y = step.ys[i].cpu().numpy()[:, rows]
        Y_ref, S = oracle_rows(wl.seed, g.w_stream, g.k, rows, X if b > 1 else X[0])
        if b == 1:
            Y_ref, S = Y_ref[None, :], S[None, :]
        worst = max(worst, assert_gemv_close(y, Y_ref, S, f"{wl.name} {g.name} b={b}"))
    return worst


@pytest.mark.parametrize("name,b", [("single_768", 1), ("minimind_26m", 1), ("minimind_26m", 2),
                                    ("minimind_26m", 8), ("minimind_26m", 16),
                                    ("smollm2_135m", 1), ("smollm2_135m", 2),
                                    ("smollm2_135m", 8), ("smollm2_135m", 16),
                                    ("gpt2_124m", 1), ("smollm2_360m", 1), ("smollm2_360m", 4),
                                    ("smollm2_135m", 12)])
def test_stack_parity(name, b):
    step = DecodeStep(synth.workloads()[name], b)
    step.run()
    torch.cuda.synchronize()
    check_step(step, 6, 100)


@pytest.mark.parametrize("b", [1, 16])
def test_graph_replay_matches_direct_launch(b):
    step = DecodeStep(synth.workloads()["smollm2_135m"], b)
    step.run()
    torch.cuda.synchronize()
    direct = [y.clone() for y in step.ys]
    for y in step.ys:
        y.fill_(float("nan"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = step.graph(s)
        g.launch(s)
        g.launch(s)
    s.synchronize()
    for a, bb in zip(direct, step.ys):
        assert torch.equal(a, bb)
    g.close()


@pytest.mark.parametrize("b", [1, 4, 16])
def test_8b_class_stack_full_size(b):
    """The benchmark's workload and launch configuration, full size, sampled rows."""
    step = DecodeStep(synth.workloads()["llama8b_class"], b)
    for _ in range(2):
        step.run()
    torch.cuda.synchronize()
    check_step(step, 4, 200)


@pytest.mark.parametrize("b", [1, 4])
def test_step_launch_count(b):
    """One kernel per dependency group, whatever the batch (the figure bench.py reports)."""
    step = DecodeStep(synth.workloads()["smollm2_135m"], b)
    step.run()
    torch.cuda.synchronize()
    c0 = q4.launch_count()
    step.run()
    torch.cuda.synchronize()
    assert q4.launch_count() - c0 == step.launches == synth.workloads()["smollm2_135m"].n_groups


def _chained_stack(d: int, f: int, layers: int, seed: int):
    """A one-token stack whose groups feed one another: per layer q, k, v read the
    previous layer's down output, o reads q, gate and up read o, down reads gate,
    and a narrow 64-row GEMV (K split across CTAs) reads down. Weights are drawn
    with std 1/sqrt(k), so activations keep their scale along the chain."""
    spec = []  # (n, k, group, source GEMV of x or -1)
    down = -1
    for layer in range(layers):
        g = 5 * layer
        q = len(spec)
        spec += [(d, d, g, down), (d // 4, d, g, down), (d // 4, d, g, down)]
        o = len(spec)
        spec.append((d, d, g + 1, q))
        gate = len(spec)
        spec += [(f, d, g + 2, o), (f, d, g + 2, o)]
        down = len(spec)
        spec.append((d, f, g + 3, gate))
        spec.append((64, d, g + 4, down))
    mats, xs, ys = [], [], []
    x0 = synth.normal(seed, 1, 0, d, 1.0, "cuda")
    for i, (n, k, _, src) in enumerate(spec):
        w = synth.normal(seed, 100 + i, 0, n * k, k ** -0.5, "cuda").view(n, k)
        mats.append(q4.pack(w))
        ys.append(torch.full((n,), float("nan"), device="cuda"))
        xs.append(x0 if src < 0 else ys[src])
    return spec, mats, xs, ys


@pytest.mark.parametrize("d,f", [(1024, 2816), (960, 2560)])
def test_chained_stack_waits_for_earlier_groups(d, f):
    """Groups that read the outputs of the group before them, over 80 groups
    (launches that start while the previous one drains, their weights streaming
    in before they wait): the step must give bit for bit the outputs of the same
    groups enqueued one call each, in direct launches and graph replays; the
    first group, whose input is synthetic, must also match the oracle."""
    spec, mats, xs, ys = _chained_stack(d, f, 16, 31)
    groups = [s[2] for s in spec]
    stack = q4.Stack(mats, xs, ys, groups)
    ws = q4.workspace(stack.workspace_bytes(1), "cuda")
    q4.layer_stack(stack, 1, ws)
    torch.cuda.synchronize()
    got = [y.clone() for y in ys]
    assert all(bool(torch.isfinite(y).all()) for y in got)
    # the same groups, one call each
    for y in ys:
        y.fill_(float("nan"))
    for g in sorted(set(groups)):
        idx = [i for i, s in enumerate(spec) if s[2] == g]
        one = q4.Stack([mats[i] for i in idx], [xs[i] for i in idx], [ys[i] for i in idx], [0] * len(idx))
        q4.layer_stack(one, 1, ws)
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(got, ys)):
        assert torch.equal(a, b), f"GEMV {i} (group {spec[i][2]}) differs from its own launch"
    # graph replays of the whole step
    for y in ys:
        y.fill_(float("nan"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gr = q4.Graph(stack, 1, ws, s)
        gr.launch(s)
        gr.launch(s)
    s.synchronize()
    for i, (a, b) in enumerate(zip(got, ys)):
        assert torch.equal(a, b), f"GEMV {i}: graph replay differs"
    gr.close()
    assert q4.workspace_status(ws) == 0
    # the first group against the oracle (its input re-drawn on the host)
    x0 = synth.normal(31, 1, 0, d, 1.0).numpy()
    assert np.array_equal(xs[0].cpu().numpy(), x0)
    for i in range(3):
        n, k = spec[i][0], spec[i][1]
        rows = sample_rows(n, 8, 7 + i)
        w = synth.matrix_rows(31, 100 + i, k, rows, k ** -0.5).numpy()
        y_ref, S = oracle.q4_gemv(oracle.q4_pack(w), len(rows), k, x0)
        assert_gemv_close(got[i].cpu().numpy()[rows], y_ref, S, f"chained GEMV {i}")
