"""Helpers shared by the GPU parity tests: moving seeded inputs to the device and running the
fp64 oracle on exactly the values the device saw."""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle
import synth

# Tolerances (relative Frobenius norm, per matrix), fixed by the benchmark spec for this path:
TOL_O_BF16 = 3e-2     # O in bf16 working precision
TOL_O_FP32 = 1e-4     # O in fp32 working precision
TOL_P = 1e-3          # updated parameters
# The momentum buffer is an fp32 EMA of fp32/bf16 inputs: a few fp32 roundings.
TOL_M = 1e-6


def rel(a: np.ndarray, b: np.ndarray) -> float:
    nb = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (nb if nb > 0 else 1.0)


def tdtype(name: str):
    return torch.bfloat16 if name == "bf16" else torch.float32


def to_dev(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype).contiguous()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


class StepCase:
    """One workload's state on the device plus the oracle's fp64 copies of sampled matrices."""

    def __init__(self, wl: synth.Workload, sample: Sequence[int], device_fill: bool = False):
        self.wl = wl
        self.sample = list(sample)
        self.params: List[torch.Tensor] = []
        self.momentum: List[torch.Tensor] = []
        gd = tdtype(wl.grad_dtype)
        for j, (r, c) in enumerate(wl.shapes):
            if device_fill and j not in self.sample:
                p = wl.param_torch(j, "cuda").to(torch.float32)
            else:
                p = to_dev(wl.param(j), torch.float32)
            self.params.append(p)
            self.momentum.append(torch.zeros((r, c), dtype=torch.float32, device="cuda"))
        self.o_params = {j: host64(self.params[j]) for j in self.sample}
        self.o_mom = {j: np.zeros(wl.shapes[j]) for j in self.sample}
        self.device_fill = device_fill
        self.gd = gd

    def grads(self, step: int) -> List[torch.Tensor]:
        out = []
        for j in range(self.wl.count):
            if self.device_fill and j not in self.sample:
                out.append(self.wl.grad_torch(j, step, "cuda").to(self.gd))
            else:
                out.append(to_dev(self.wl.grad(j, step), self.gd))
        return out

    def step(self, step: int, prec: str = "bf16", coeffs=None):
        import newton_schulz_13_b200 as ns
        wl = self.wl
        co = coeffs or wl.coeffs
        g = self.grads(step)
        ns.muon_step(self.params, g, self.momentum, lr=wl.lr, mu=wl.mu, nesterov=wl.nesterov,
                     weight_decay=wl.weight_decay, rms_scale=wl.rms_scale, steps=len(co), coeffs=co,
                     zero_center=wl.zero_center, eps=wl.eps, prec=prec)
        O = {}
        for j in self.sample:
            gj = host64(g[j])
            O[j] = oracle.muon_step([self.o_params[j]], [gj], [self.o_mom[j]], lr=wl.lr, mu=wl.mu,
                                    nesterov=wl.nesterov, weight_decay=wl.weight_decay,
                                    rms_mode=wl.rms_scale, coeffs=co, zero_center=wl.zero_center,
                                    eps=wl.eps, want_O=True)[0]
        return g, O

    def rms(self, j: int) -> float:
        r, c = self.wl.shapes[j]
        return float(np.sqrt(max(1.0, r / c))) if self.wl.rms_scale == 1 else 1.0
