"""Decode steps (layer stacks) on the GPU against the oracle, on sampled rows of
every GEMV; direct launches and graph replays must agree bit for bit."""
import numpy as np
import pytest
import torch

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
