"""Seeded synthetic inputs for the MoE layer (shared by the tests and the benchmark).

This module holds no arithmetic of the layer itself: it only draws inputs.
Both the CUDA path and the CPU oracle are fed the same tensors from here.

Generator (counter-based, so any element can be drawn independently and the
result does not depend on the device or the chunking):

  key(seed, tag)  = mix64(seed * 2^32 + tag)
  z_i             = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)      (mod 2^64)
  mix64(x)        = splitmix64 finaliser:
                      x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9
                      x = (x ^ (x >> 27)) * 0x94D049BB133111EB
                      x =  x ^ (x >> 31)
  u1 = ((z_i >> 32) + 0.5) / 2^32,  u2 = (z_i & 0xffffffff) / 2^32
  n_i = sqrt(-2 ln u1) * cos(2 pi u2)                               (Box-Muller, fp64)

then scaled by the standard deviation and rounded to nearest-even bf16 (x and
the weights) or fp32 (gate logits).  Tags: x=1, logits=2, W1=3, W3=4, W2=5,
per-expert router bias=6.

Workloads: the layer shapes and router distributions of the synthetic
benchmark suite (a tiny layer, a Mixtral-8x7B-shaped layer, a fine-grained
64-expert layer, a 128-expert imbalanced layer and a d=4096/E=32/top-4 sweep).
Router biases: "zipf" gives expert e the bias -1.5 * 1.2 * ln(e + 1) (rank e+1 of
a Zipf(s=1.2) law, times 1.5); "normal2" draws one N(0, 2) bias per expert;
"hot" adds +6 to expert 0.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

TAG_X, TAG_LOGITS, TAG_W1, TAG_W3, TAG_W2, TAG_BIAS = 1, 2, 3, 4, 5, 6


def _s64(v: int) -> int:
    """uint64 bit pattern -> the int64 with the same bits."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix64_int(x: int) -> int:
    x &= _MASK64
    x = ((x ^ (x >> 30)) * _M1) & _MASK64
    x = ((x ^ (x >> 27)) * _M2) & _MASK64
    return x ^ (x >> 31)


def key(seed: int, tag: int) -> int:
    return _mix64_int(((seed & 0xFFFFFFFF) << 32) | (tag & 0xFFFFFFFF))


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    # logical right shift on the int64 bit pattern
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def raw64(seed: int, tag: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """z_i for i in [start, start+count), as int64 tensors holding the uint64 bits."""
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = i * _s64(_GAMMA) + _s64(key(seed, tag))
    return _mix64(z)


def normal(seed: int, tag: int, n: int, std: float = 1.0, device="cpu",
           dtype=torch.bfloat16, chunk: int = 1 << 24) -> torch.Tensor:
    """n draws of N(0, std^2), rounded to `dtype` (RNE)."""
    out = torch.empty(n, dtype=dtype, device=device)
    two32 = float(1 << 32)
    for s in range(0, n, chunk):
        c = min(chunk, n - s)
        z = raw64(seed, tag, s, c, device)
        hi = _lsr(z, 32).to(torch.float64)
        lo = (z & 0xFFFFFFFF).to(torch.float64)
        u1 = (hi + 0.5) / two32
        u2 = lo / two32
        v = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
        out[s:s + c] = (v * std).to(dtype)
        del z, hi, lo, u1, u2, v
    return out


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    f: int
    E: int
    k: int
    router: str = "uniform"       # uniform | zipf | normal2 | hot
    seed: int = 0x5EED0000
    x_std: float = 1.0
    w_std: float = 0.02
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def R(self) -> int:
        return self.T * self.k

    def flops(self) -> int:
        """Algorithmic FLOPs of the expert FFN: 6 * T*k * d * f (no masked rows)."""
        return 6 * self.R * self.d * self.f


def _sweep():
    res = {}
    for ti, T in enumerate((512, 2048, 8192, 32768)):
        for ri, router in enumerate(("uniform", "zipf", "hot")):
            name = f"sweep_T{T}_{router}"
            res[name] = Workload(name, T, 4096, 2048, 32, 4, router,
                                 0x5EED0000 + 4 + 100 * ti + 10 * ri)
    return res


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 256, 512, 1024, 8, 2, "uniform", 0x5EED0000 + 0),
    "mixtral": Workload("mixtral", 4096, 4096, 14336, 8, 2, "uniform", 0x5EED0000 + 1),
    "fine_grained": Workload("fine_grained", 8192, 2048, 1408, 64, 6, "zipf", 0x5EED0000 + 2),
    "imbalanced": Workload("imbalanced", 16384, 4096, 1536, 128, 8, "normal2", 0x5EED0000 + 3),
    # a profiling case of the Mixtral-shaped layer: the same expert shape and rows per
    # expert (1024) with 2 experts instead of 8, about a quarter of the device memory
    "mixtral_e2": Workload("mixtral_e2", 1024, 4096, 14336, 2, 2, "uniform", 0x5EED0000 + 5),
    **_sweep(),
}


def router_bias(wl: Workload, device="cpu") -> torch.Tensor:
    E = wl.E
    if wl.router == "uniform":
        return torch.zeros(E, dtype=torch.float64, device=device)
    if wl.router == "zipf":
        e = torch.arange(E, dtype=torch.float64, device=device)
        return -1.5 * 1.2 * torch.log(e + 1.0)
    if wl.router == "normal2":
        return normal(wl.seed, TAG_BIAS, E, 2.0, device, torch.float64)
    if wl.router == "hot":
        b = torch.zeros(E, dtype=torch.float64, device=device)
        b[0] = 6.0
        return b
    raise ValueError(f"unknown router mode {wl.router!r}")


def make_logits(wl: Workload, device="cpu") -> torch.Tensor:
    z = normal(wl.seed, TAG_LOGITS, wl.T * wl.E, 1.0, device, torch.float64).view(wl.T, wl.E)
    return (z + router_bias(wl, device)[None, :]).to(torch.float32)


def make_x(wl: Workload, device="cpu") -> torch.Tensor:
    return normal(wl.seed, TAG_X, wl.T * wl.d, wl.x_std, device).view(wl.T, wl.d)


def make_weights(wl: Workload, device="cpu"):
    """W1, W3: [E][d][f]; W2: [E][f][d]; bf16 ~ N(0, w_std^2)."""
    n = wl.E * wl.d * wl.f
    W1 = normal(wl.seed, TAG_W1, n, wl.w_std, device).view(wl.E, wl.d, wl.f)
    W3 = normal(wl.seed, TAG_W3, n, wl.w_std, device).view(wl.E, wl.d, wl.f)
    W2 = normal(wl.seed, TAG_W2, n, wl.w_std, device).view(wl.E, wl.f, wl.d)
    return W1, W3, W2


def make_inputs(wl: Workload, device="cpu", weights: bool = True) -> dict:
    res = dict(x=make_x(wl, device), logits=make_logits(wl, device))
    if weights:
        res["W1"], res["W3"], res["W2"] = make_weights(wl, device)
    return res


def small(name: str, T: int, d: int, f: int, E: int, k: int, router: str = "uniform",
          seed: int = 1234) -> Workload:
    """An ad-hoc workload for tests (same generator, other shapes)."""
    return Workload(name, T, d, f, E, k, router, seed)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def from_bf16_bits(a) -> torch.Tensor:
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
