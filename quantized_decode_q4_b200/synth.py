"""Seeded synthetic inputs and the decode workloads they fill.

This module is shared by the tests, the benchmark and the oracle side of the
parity checks. It holds no Q4_0 arithmetic: it only draws binary32 numbers and
lists matrix shapes.

Generator (counter based, so any element range can be drawn on its own, on
the host or on the GPU, with identical bits):
  * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state_n = key + (n + 1) * 0x9E3779B97F4A7C15 mod
    2^64, output_n = mix(state_n), with the published 64-bit finaliser
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
    z ^= z >> 31.
  * key = mix((seed << 32) | stream), one stream per tensor.
  * An approximately standard normal value is the textbook Irwin-Hall sum of
    twelve uniforms minus six: element i uses outputs 12 i .. 12 i + 11, keeps
    the top 24 bits u_j of each, and returns (sum_j u_j - 6 (2^24 - 1)) / 2^24,
    formed exactly in binary64 and rounded once to binary32, then multiplied by
    the binary32 standard deviation (one binary32 rounding).
Only integer operations precede the two roundings, so torch on the CPU, torch
on the GPU and the numpy twin all give the same bits.

Workloads follow the model shapes the pages name: GPT-2 124M, SmolLM2 135M and
360M, MiniMind 26M ("MicroLLM Lab", "Seven models, all in Q4") and an 8B-class
Llama layer ("gputps.com" catalogue, 8B sizing paragraph).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1
UNIFORMS_PER_NORMAL = 12
CENTER = 6 * ((1 << 24) - 1)


def _signed(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _signed(MIX1)
    z = (z ^ _lsr(z, 27)) * _signed(MIX2)
    return z ^ _lsr(z, 31)


def _mix_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    if not (0 <= seed < 2**31 and 0 <= stream < 2**32):
        raise ValueError("seed must be < 2^31 and stream < 2^32")
    return _mix_int((seed << 32) | stream)


def normal(seed: int, stream: int, start: int, count: int, std: float = 1.0,
           device="cpu", chunk: int = 1 << 22) -> torch.Tensor:
    """Elements start .. start+count-1 of stream `stream` as binary32 N(0, std^2)."""
    key = stream_key(seed, stream)
    out = torch.empty(count, dtype=torch.float32, device=device)
    std_t = torch.tensor(std, dtype=torch.float32, device=device)
    j = torch.arange(UNIFORMS_PER_NORMAL, dtype=torch.int64, device=device)
    for c0 in range(0, count, chunk):
        c1 = min(count, c0 + chunk)
        i = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
        n = i[:, None] * UNIFORMS_PER_NORMAL + j[None, :] + 1
        state = n * _signed(GAMMA) + _signed(key)
        u = _lsr(_mix_t(state), 40)
        s = u.sum(dim=1) - CENTER
        z = (s.to(torch.float64) * (2.0 ** -24)).to(torch.float32)
        out[c0:c1] = z * std_t
        del n, state, u, s, z
    return out


def normal_np(seed: int, stream: int, start: int, count: int, std: float = 1.0) -> np.ndarray:
    """numpy twin of `normal` (uint64 arithmetic), used to cross-check the torch form."""
    key = np.uint64(stream_key(seed, stream))
    i = np.arange(start, start + count, dtype=np.uint64)
    n = i[:, None] * np.uint64(UNIFORMS_PER_NORMAL) + np.arange(
        UNIFORMS_PER_NORMAL, dtype=np.uint64)[None, :] + np.uint64(1)
    with np.errstate(over="ignore"):
        z = n * np.uint64(GAMMA) + key
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
        z = z ^ (z >> np.uint64(31))
    u = (z >> np.uint64(40)).astype(np.int64)
    s = u.sum(axis=1) - CENTER
    zf = (s.astype(np.float64) * (2.0 ** -24)).astype(np.float32)
    return zf * np.float32(std)


def matrix(seed: int, stream: int, n: int, k: int, std: float, device="cpu") -> torch.Tensor:
    return normal(seed, stream, 0, n * k, std, device).view(n, k)


def matrix_rows(seed: int, stream: int, k: int, rows, std: float, device="cpu") -> torch.Tensor:
    """Selected rows of `matrix(seed, stream, n, k, std)` without drawing the rest."""
    rows = list(int(r) for r in rows)
    out = torch.empty(len(rows), k, dtype=torch.float32, device=device)
    for i, r in enumerate(rows):
        out[i] = normal(seed, stream, r * k, k, std, device)
    return out


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

WEIGHT_STD = 0.02
ACT_STD = 1.0


@dataclass
class Gemv:
    """One Q4_0 matrix-vector product of a decode step."""
    name: str
    n: int                 # output rows
    k: int                 # inputs (multiple of 32)
    group: int             # dependency group: groups run in order, members together
    w_stream: int          # generator stream of the binary32 weights
    x_stream: int          # generator stream of the activations [batch][k]

    @property
    def q4_bytes(self) -> int:
        return self.n * self.k * 18 // 32


@dataclass
class Workload:
    name: str
    seed: int
    gemvs: list = field(default_factory=list)
    batches: tuple = (1,)

    @property
    def q4_bytes(self) -> int:
        return sum(g.q4_bytes for g in self.gemvs)

    @property
    def n_groups(self) -> int:
        return len({g.group for g in self.gemvs})

    def weights(self, i: int, device="cpu") -> torch.Tensor:
        g = self.gemvs[i]
        return matrix(self.seed, g.w_stream, g.n, g.k, WEIGHT_STD, device)

    def activations(self, i: int, batch: int, device="cpu") -> torch.Tensor:
        g = self.gemvs[i]
        return normal(self.seed, g.x_stream, 0, batch * g.k, ACT_STD, device).view(batch, g.k)


def _stack(name, seed, layers, per_layer_groups, head=None, batches=(1,), stream_base=0):
    """per_layer_groups: list of groups, each a list of (name, n, k)."""
    wl = Workload(name, seed, batches=batches)
    t = 0
    group = 0
    for layer in range(layers):
        for members in per_layer_groups:
            for (nm, n, k) in members:
                s = stream_base + 2 * t
                wl.gemvs.append(Gemv(f"L{layer}.{nm}", n, k, group, s, s + 1))
                t += 1
            group += 1
    if head is not None:
        s = stream_base + 2 * t
        wl.gemvs.append(Gemv("head", head[0], head[1], group, s, s + 1))
    return wl


def _llama_groups(d, q_rows, kv_rows, ffn):
    return [[("q", q_rows, d), ("k", kv_rows, d), ("v", kv_rows, d)],
            [("o", d, q_rows)],
            [("gate", ffn, d), ("up", ffn, d)],
            [("down", d, ffn)]]


def workloads() -> dict:
    """The synthetic decode steps, keyed by name."""
    w = {}
    w["single_768"] = _stack("single_768", 0, 1, [[("w", 768, 768)]])
    w["gpt2_124m"] = _stack(
        "gpt2_124m", 1, 12,
        [[("qkv", 2304, 768)], [("proj", 768, 768)], [("fc", 3072, 768)],
         [("fc_proj", 768, 3072)]],
        head=(50257, 768))
    w["smollm2_360m"] = _stack("smollm2_360m", 2, 32, _llama_groups(960, 960, 320, 2560),
                               head=(49152, 960), batches=(1, 4))
    w["minimind_26m"] = _stack("minimind_26m", 3, 8, _llama_groups(512, 512, 128, 1408),
                               batches=(1, 2, 8, 16))
    w["smollm2_135m"] = _stack("smollm2_135m", 3, 30, _llama_groups(576, 576, 192, 1536),
                               head=(49152, 576), batches=(1, 2, 8, 16), stream_base=1 << 20)
    w["llama8b_class"] = _stack("llama8b_class", 4, 32, _llama_groups(4096, 4096, 1024, 14336),
                                batches=(1, 4))
    return w
