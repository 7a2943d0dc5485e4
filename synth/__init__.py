"""Seeded synthetic inputs for the Muon step: workload definitions and generators.

This module is shared by the fp64 oracle, the parity tests and the benchmark.
It holds none of the method's arithmetic (no momentum, normalisation,
Newton-Schulz or update): only the shapes, hyper-parameters and random draws
of each workload.

Generator (counter based, so any matrix can be regenerated alone, on the host
or on a device, without generating the ones before it):

* ``mix`` is the splitmix64 output function (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014).
* A matrix is keyed by ``(seed, matrix index, kind, step)``; element ``e`` of
  it draws two 64-bit words ``mix(key + (2e+1)*GAMMA)`` and
  ``mix(key + (2e+2)*GAMMA)`` (the splitmix64 stream started at ``key``),
  turns each into a uniform double in (0, 1) from its top 53 bits, and maps
  the pair to one standard normal by the Box-Muller cosine branch.
* Per-column scales ``s_j = exp(ln lo + U_j (ln hi - ln lo))`` (log-uniform on
  [lo, hi]) use their own key kind, so they do not depend on the step.

Values are produced in float64 and rounded once to the workload's storage
dtype (fp32 or bf16) by the caller; the oracle consumes the rounded values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_K_SEED = 0xD1B54A32D192ED03
_K_MAT = 0xABC98388FB8FAC03
_K_KIND = 0x8CB92BA72F3D8DD7
_K_STEP = 0xC6A4A7935BD1E995
_MASK64 = (1 << 64) - 1

KIND_GRAD = 1
KIND_PARAM = 2
KIND_COLSCALE = 3

QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def matrix_key(seed: int, mat: int, kind: int, step: int) -> int:
    """64-bit key of one generated matrix (pure integer hashing)."""
    z = (seed * _K_SEED + (mat + 1) * _K_MAT + kind * _K_KIND + (step + 1) * _K_STEP) & _MASK64
    return _mix_int(_mix_int(z))


# ----------------------------------------------------------------------------
# numpy backend (host)
# ----------------------------------------------------------------------------

def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def _uniform_np(key: int, n: int, which: int, stride: int = 2) -> np.ndarray:
    """Uniform doubles in (0,1): word ``stride*e + which + 1`` of the stream at ``key``."""
    with np.errstate(over="ignore"):
        e = np.arange(n, dtype=np.uint64)
        z = np.uint64(key) + (e * np.uint64(stride) + np.uint64(which + 1)) * np.uint64(GAMMA)
        w = _mix_np(z)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def standard_normal(key: int, n: int) -> np.ndarray:
    u1 = _uniform_np(key, n, 0)
    u2 = _uniform_np(key, n, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def log_uniform(key: int, n: int, lo: float, hi: float) -> np.ndarray:
    u = _uniform_np(key, n, 0, stride=1)
    return np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))


# ----------------------------------------------------------------------------
# torch backend (same integer stream; used to fill large device buffers)
# ----------------------------------------------------------------------------

def _signed(c: int) -> int:
    c &= _MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


def _lsr_t(x, s: int):
    import torch
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z):
    z = (z ^ _lsr_t(z, 30)) * _signed(_M1)
    z = (z ^ _lsr_t(z, 27)) * _signed(_M2)
    return z ^ _lsr_t(z, 31)


def _uniform_t(key: int, n: int, which: int, device, stride: int = 2):
    import torch
    e = torch.arange(n, dtype=torch.int64, device=device)
    z = _signed(key) + (e * stride + (which + 1)) * _signed(GAMMA)
    w = _mix_t(z)
    return (_lsr_t(w, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def standard_normal_torch(key: int, n: int, device):
    import torch
    u1 = _uniform_t(key, n, 0, device)
    u2 = _uniform_t(key, n, 1, device)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)


def log_uniform_torch(key: int, n: int, lo: float, hi: float, device):
    import torch
    u = _uniform_t(key, n, 0, device, stride=1)
    return torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass
class Dist:
    """N(0, std^2), optionally times a per-column log-uniform scale on [lo, hi]."""
    std: float = 1.0
    colscale: Optional[Tuple[float, float]] = None


@dataclass
class Workload:
    name: str
    description: str
    shapes: List[Tuple[int, int]]
    grad_dtype: str                 # "fp32" or "bf16"
    grad_dist: Dist
    param_std: float
    seed: int
    coeffs: List[Tuple[float, float, float]]
    lr: float
    mu: float
    nesterov: bool
    weight_decay: float
    rms_scale: int                  # 0: none, 1: sqrt(max(1, rows/cols))
    zero_center: bool
    eps: float
    n_steps: int                    # optimizer steps of the parity run
    layer_size: int = 1             # matrices per layer (for sampling whole layers)

    @property
    def count(self) -> int:
        return len(self.shapes)

    def grad(self, mat: int, step: int) -> np.ndarray:
        r, c = self.shapes[mat]
        z = standard_normal(matrix_key(self.seed, mat, KIND_GRAD, step), r * c).reshape(r, c)
        z *= self.grad_dist.std
        if self.grad_dist.colscale is not None:
            lo, hi = self.grad_dist.colscale
            z *= log_uniform(matrix_key(self.seed, mat, KIND_COLSCALE, 0), c, lo, hi)[None, :]
        return z

    def param(self, mat: int) -> np.ndarray:
        r, c = self.shapes[mat]
        return standard_normal(matrix_key(self.seed, mat, KIND_PARAM, 0), r * c).reshape(r, c) * self.param_std

    def grad_torch(self, mat: int, step: int, device):
        r, c = self.shapes[mat]
        z = standard_normal_torch(matrix_key(self.seed, mat, KIND_GRAD, step), r * c, device).view(r, c)
        z *= self.grad_dist.std
        if self.grad_dist.colscale is not None:
            lo, hi = self.grad_dist.colscale
            z *= log_uniform_torch(matrix_key(self.seed, mat, KIND_COLSCALE, 0), c, lo, hi, device)[None, :]
        return z

    def param_torch(self, mat: int, device):
        r, c = self.shapes[mat]
        return standard_normal_torch(matrix_key(self.seed, mat, KIND_PARAM, 0), r * c, device).view(r, c) * self.param_std

    def ns_flops(self) -> float:
        """Nominal Newton-Schulz FLOPs of one step: per iteration 4 m^2 n + 2 m^3
        (m = min dim, n = max dim); 4 m^2 n when the A^2 term is absent (c = 0)."""
        tot = 0.0
        for (r, c) in self.shapes:
            m, n = min(r, c), max(r, c)
            for (_, _, cc) in self.coeffs:
                tot += 4.0 * m * m * n + (2.0 * m ** 3 if cc != 0.0 else 0.0)
        return tot

    def elements(self) -> int:
        return sum(r * c for r, c in self.shapes)


def _rep(block: Sequence[Tuple[int, int]], n: int) -> List[Tuple[int, int]]:
    return [s for _ in range(n) for s in block]


WORKLOADS = {
    "single_256x512": Workload(
        name="single_256x512",
        description="one 256x512 fp32 gradient N(0,1), seed 0, zero momentum, Nesterov mu=0.95, "
                    "quintic x5, eps 1e-7, lr 0.02, one step",
        shapes=[(256, 512)], grad_dtype="fp32", grad_dist=Dist(1.0), param_std=0.02, seed=0,
        coeffs=[QUINTIC] * 5, lr=0.02, mu=0.95, nesterov=True, weight_decay=0.0, rms_scale=0,
        zero_center=False, eps=1e-7, n_steps=1),
    "cubic_zero_center_12": Workload(
        name="cubic_zero_center_12",
        description="cubic NS x5 with zero-centering along dim 0: 6 x 768x768 and 6 x 768x3072 fp32 "
                    "gradients N(0,1) x column scale log-uniform [1e-4,1e-1], seed 1",
        shapes=[(768, 768)] * 6 + [(768, 3072)] * 6, grad_dtype="fp32",
        grad_dist=Dist(1.0, (1e-4, 1e-1)), param_std=0.02, seed=1,
        coeffs=[CUBIC] * 5, lr=0.02, mu=0.95, nesterov=True, weight_decay=0.0, rms_scale=0,
        zero_center=True, eps=1e-7, n_steps=1),
    "gpt2_small": Workload(
        name="gpt2_small",
        description="GPT-2-small hidden weights, 12 layers x {768x2304, 768x768, 768x3072, 3072x768}, "
                    "bf16 grads N(0,1e-3) x column scale [0.1,10], fp32 params N(0,0.02), quintic x5, "
                    "mu 0.95, lr 0.02, wd 0.01, 10 consecutive steps",
        shapes=_rep([(768, 2304), (768, 768), (768, 3072), (3072, 768)], 12), grad_dtype="bf16",
        grad_dist=Dist(1e-3, (0.1, 10.0)), param_std=0.02, seed=3,
        coeffs=[QUINTIC] * 5, lr=0.02, mu=0.95, nesterov=True, weight_decay=0.01, rms_scale=0,
        zero_center=False, eps=1e-7, n_steps=10, layer_size=4),
    "mamba_24": Workload(
        name="mamba_24",
        description="Mamba blocks, 24 layers x {in_proj 3072x768, x_proj 80x1536, dt_proj 1536x48, "
                    "out_proj 768x1536}, bf16 grads N(0,1e-3) x column scale [0.1,10], quintic x5, "
                    "Nesterov mu 0.95, 3 steps",
        shapes=_rep([(3072, 768), (80, 1536), (1536, 48), (768, 1536)], 24), grad_dtype="bf16",
        grad_dist=Dist(1e-3, (0.1, 10.0)), param_std=0.02, seed=4,
        coeffs=[QUINTIC] * 5, lr=0.02, mu=0.95, nesterov=True, weight_decay=0.0, rms_scale=0,
        zero_center=False, eps=1e-7, n_steps=3, layer_size=4),
    "llama8b": Workload(
        name="llama8b",
        description="Llama-8B hidden weights, 32 layers x {Wq 4096x4096, Wk 1024x4096, Wv 1024x4096, "
                    "Wo 4096x4096, gate 14336x4096, up 14336x4096, down 4096x14336}, bf16 grads N(0,1) x "
                    "column scale [1e-4,1e-1], fp32 params N(0,0.02), quintic x5, lr 0.02, wd 0.1, "
                    "RMS rescale sqrt(max(1, rows/cols))",
        shapes=_rep([(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096),
                     (14336, 4096), (14336, 4096), (4096, 14336)], 32), grad_dtype="bf16",
        grad_dist=Dist(1.0, (1e-4, 1e-1)), param_std=0.02, seed=5,
        coeffs=[QUINTIC] * 5, lr=0.02, mu=0.95, nesterov=True, weight_decay=0.1, rms_scale=1,
        zero_center=False, eps=1e-7, n_steps=1, layer_size=7),
}

# One layer of the Llama-8B set (7 matrices, 2.2e8 elements): a few GB on the device, still
# larger than L2, used for detailed kernel profiles.
WORKLOADS["llama8b_layer"] = Workload(**{**WORKLOADS["llama8b"].__dict__, "name": "llama8b_layer",
                                         "description": "one layer of the Llama-8B hidden-weight set",
                                         "shapes": WORKLOADS["llama8b"].shapes[:7]})

# ----------------------------------------------------------------------------
# AdamW workloads: the parameters that do not go to Muon (embeddings, head, norms, biases)
# ----------------------------------------------------------------------------

@dataclass
class AdamWorkload:
    name: str
    description: str
    sizes: List[int]                # numel of each tensor
    grad_dtype: str
    grad_std: float
    param_std: float
    seed: int
    lr: float
    beta1: float
    beta2: float
    eps: float
    weight_decay: float
    n_steps: int

    @property
    def count(self) -> int:
        return len(self.sizes)

    def elements(self) -> int:
        return sum(self.sizes)

    def grad(self, i: int, step: int) -> np.ndarray:
        return standard_normal(matrix_key(self.seed, i, KIND_GRAD, step), self.sizes[i]) * self.grad_std

    def param(self, i: int) -> np.ndarray:
        return standard_normal(matrix_key(self.seed, i, KIND_PARAM, 0), self.sizes[i]) * self.param_std

    def grad_torch(self, i: int, step: int, device):
        return standard_normal_torch(matrix_key(self.seed, i, KIND_GRAD, step), self.sizes[i], device) * self.grad_std

    def param_torch(self, i: int, device):
        return standard_normal_torch(matrix_key(self.seed, i, KIND_PARAM, 0), self.sizes[i], device) * self.param_std


_GPT2_SMALL_ADAM = ([50257 * 768, 1024 * 768]                             # token and position embeddings
                    + [768, 768, 2304, 768, 768, 768, 3072, 768] * 12     # per layer: ln1 w/b, qkv b, proj b,
                    + [768, 768])                                          # ln2 w/b, fc b, fc-proj b; final ln
_LLAMA8B_ADAM = [128256 * 4096, 128256 * 4096] + [4096] * 65               # embedding, head, 2 norms x 32 + final

ADAM_WORKLOADS = {
    "gpt2_small_adamw": AdamWorkload(
        name="gpt2_small_adamw",
        description="GPT-2-small parameters outside Muon: embeddings, layer-norm scales and shifts, biases",
        sizes=_GPT2_SMALL_ADAM, grad_dtype="bf16", grad_std=1e-3, param_std=0.02, seed=13, lr=1e-3,
        beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01, n_steps=3),
    "llama8b_adamw": AdamWorkload(
        name="llama8b_adamw",
        description="Llama-8B parameters outside Muon: token embedding and prediction head (128256 x 4096), "
                    "65 RMSNorm scales of 4096",
        sizes=_LLAMA8B_ADAM, grad_dtype="bf16", grad_std=1.0, param_std=0.02, seed=15, lr=1e-3,
        beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, n_steps=1),
}

# The eight-plus-two coefficient schedule (eight quintic iterations, then two
# with (2, -1.5, 0.5)), exercised on the GPT-2-small shapes.
HYBRID = [(3.445, -4.7750, 2.0315)] * 8 + [(2.0, -1.5, 0.5)] * 2


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values once to the storage dtype and return them as float64."""
    if dtype == "fp32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        import torch
        return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()
    raise ValueError(dtype)
