"""A synthetic decode step on the GPU: packed weights, activations, outputs, workspace.

Weights of every GEMV are drawn on the device by the seeded generator and packed
by the library's q4_pack kernel; the binary32 copy is dropped right after packing,
so only the Q4_0 planes (4.5 bits per weight) stay resident.
"""
from __future__ import annotations

import torch

from . import _lib as q4
from . import synth


def _pad4(v: int) -> int:
    return (v + 3) // 4 * 4


class DecodeStep:
    """All activations live in one device buffer and all outputs in another (each
    GEMV's slice starts on a 16-byte boundary), so a step's inputs and results move
    between host and device with one copy each."""

    def __init__(self, workload: synth.Workload, batch: int, device="cuda", mats=None):
        """mats: the packed weights of another step of the same workload to share
        (the weights do not depend on the batch); drawn and packed here if None."""
        self.workload, self.batch, self.device = workload, batch, device
        self.mats, groups = [], []
        x_off, y_off, xo, yo = [], [], 0, 0
        for g in workload.gemvs:
            x_off.append(xo)
            y_off.append(yo)
            xo += _pad4(batch * g.k)
            yo += _pad4(batch * g.n)
        self.x_all = torch.empty(xo, dtype=torch.float32, device=device)
        self.y_all = torch.empty(yo, dtype=torch.float32, device=device)
        self.xs, self.ys = [], []
        for i, g in enumerate(workload.gemvs):
            if mats is not None:
                self.mats.append(mats[i])
            else:
                w = synth.normal(workload.seed, g.w_stream, 0, g.n * g.k, synth.WEIGHT_STD, device,
                                 chunk=1 << 24).view(g.n, g.k)
                self.mats.append(q4.pack(w))
                del w
            x = self.x_all[x_off[i]: x_off[i] + batch * g.k].view(batch, g.k)
            x.copy_(synth.normal(workload.seed, g.x_stream, 0, batch * g.k, synth.ACT_STD,
                                 device).view(batch, g.k))
            self.xs.append(x)
            self.ys.append(self.y_all[y_off[i]: y_off[i] + batch * g.n].view(batch, g.n))
            groups.append(g.group)
        self.groups = groups
        self.stack = q4.Stack(self.mats, self.xs, self.ys, groups)
        self.ws = q4.workspace(self.stack.workspace_bytes(batch), device)
        torch.cuda.synchronize()

    @property
    def x_bytes(self) -> int:
        return sum(x.numel() for x in self.xs) * 4

    @property
    def y_bytes(self) -> int:
        return sum(y.numel() for y in self.ys) * 4

    @property
    def algorithmic_bytes(self) -> int:
        """Bytes a step must move at least: Q4_0 weights once, x and y once each."""
        return self.q4_bytes + self.x_bytes + self.y_bytes

    @property
    def q4_bytes(self) -> int:
        return sum(m.nbytes for m in self.mats)

    @property
    def launches(self) -> int:
        """Kernels one step launches: one per dependency group (batch 1 on the CUDA
        cores, 2..16 tokens on the tensor cores, all tokens in one launch)."""
        return self.workload.n_groups

    def weight_copies(self, r: int) -> list:
        """r stacks of this step (this one first), the others over byte-identical
        copies of the packed weights at other addresses, with the same activations
        and outputs: running them in turn reads r different weight sets, so a set
        that fits in L2 is still streamed from HBM when r copies exceed it."""
        stacks = [self.stack]
        self._copies = []
        for _ in range(r - 1):
            mats = [q4.Q4Matrix(m.n, m.k, qs=m.qs.clone(), d=m.d.clone()) for m in self.mats]
            self._copies.append(mats)
            stacks.append(q4.Stack(mats, self.xs, self.ys, self.groups))
        return stacks

    def run(self, stream=None):
        q4.layer_stack(self.stack, self.batch, self.ws, stream)

    def graph(self, stream) -> q4.Graph:
        return q4.Graph(self.stack, self.batch, self.ws, stream)
