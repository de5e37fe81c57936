"""The seeded input generator: torch and numpy forms agree, ranges are independent."""
import numpy as np
import torch

from quantized_decode_q4_b200 import synth


def test_torch_matches_numpy_twin():
    a = synth.normal(3, 17, 1000, 50000, 0.02).numpy()
    b = synth.normal_np(3, 17, 1000, 50000, 0.02)
    assert a.view(np.uint32).tolist() == b.view(np.uint32).tolist()


def test_ranges_and_rows_are_independent():
    full = synth.matrix(1, 4, 40, 96, 0.02)
    rows = synth.matrix_rows(1, 4, 96, [0, 7, 39], 0.02)
    assert torch.equal(rows, full[[0, 7, 39]])
    small = synth.normal(1, 4, 0, 100, 0.02, chunk=7)
    assert torch.equal(small, full.view(-1)[:100])


def test_streams_differ_and_moments():
    a = synth.normal(0, 0, 0, 200000, 1.0)
    b = synth.normal(0, 1, 0, 200000, 1.0)
    assert not torch.equal(a, b)
    assert abs(a.mean().item()) < 0.01 and abs(a.std().item() - 1.0) < 0.01
    w = synth.normal(2, 9, 0, 200000, 0.02)
    assert abs(w.std().item() - 0.02) < 0.0003
    assert a.abs().max().item() <= 6.0


def test_workload_streams_unique():
    for wl in synth.workloads().values():
        streams = [s for g in wl.gemvs for s in (g.w_stream, g.x_stream)]
        assert len(streams) == len(set(streams))
        groups = [g.group for g in wl.gemvs]
        assert groups == sorted(groups)
        assert all(g.k % 32 == 0 for g in wl.gemvs)
