"""Closed-form size facts the pages fix, checked on the oracle's packed output.

"MicroLLM Lab" (sitech.ge), "Seven models, all in Q4": 16-bit weights become 4 bits
per parameter, about 75% less memory; models above 100M parameters fit in 50-84 MB.
gputps.com catalogue, parameter-count paragraph: 8B parameters take 16 GB at two bytes
each and "closer to five" GB at about four bits; its efficiency paragraph: four or
five bits instead of sixteen cut memory by about three quarters.
"""
import numpy as np

import oracle
from quantized_decode_q4_b200 import synth


def test_block_size_and_bits_per_parameter(oracle_lib):
    for n, k in [(1, 32), (3, 96), (7, 960), (2, 1408)]:
        blocks = oracle.q4_pack(np.zeros((n, k), np.float32))
        assert blocks.nbytes == n * k * 18 // 32
        assert blocks.nbytes * 8 / (n * k) == 4.5


def test_memory_reduction_versus_16_bit():
    codes_only = 1 - 4 / 16
    with_scales = 1 - 4.5 / 16
    assert codes_only == 0.75          # the pages' "about 75%" is the codes alone
    assert with_scales == 0.71875      # the scale per 32 weights costs 0.5 bit each


def test_8b_model_sizes():
    params = 8.0e9
    assert params * 2 == 16e9                       # 16 GB at two bytes per parameter
    q4 = params * 18 / 32
    assert q4 == 4.5e9 and q4 < 5e9                 # "closer to five" GB at ~4 bits


def test_workload_q4_bytes():
    w = synth.workloads()
    expect_mb = {"single_768": 0.331776, "gpt2_124m": 69.486768, "smollm2_360m": 203.48928,
                 "minimind_26m": 12.681216, "smollm2_135m": 75.644928,
                 "llama8b_class": 3925.868544}
    for name, mb in expect_mb.items():
        assert abs(w[name].q4_bytes / 1e6 - mb) < 1e-9
        assert w[name].q4_bytes == sum(g.n * g.k for g in w[name].gemvs) * 9 // 16
    # a 135M-class Q4_0 stack sits inside the 50-84 MB range quoted for >100M models
    assert 50e6 <= w["smollm2_135m"].q4_bytes <= 84e6
    # gemv counts per decode step
    assert [len(w[n].gemvs) for n in ("gpt2_124m", "smollm2_360m", "minimind_26m",
                                      "smollm2_135m", "llama8b_class")] == [49, 225, 56, 211, 224]
