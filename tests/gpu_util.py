"""Helpers for the GPU parity tests: seeded inputs on the device, host copies
for the oracle, and the comparison rules.

Tolerance for bf16 outputs (fp32 accumulation): max |gpu - oracle| <=
2e-2 * max |oracle| over the compared elements.  Integer routing outputs
(top-k ids, counts, offsets, permutation) must match exactly; gates within
1e-6 relative (both sides compute them in double and round to fp32)."""
from __future__ import annotations

import numpy as np
import torch

from combine_overlap_b200 import synth

REL_TOL = 2e-2


def inputs(wl: synth.Workload, device="cuda", weights=True) -> dict:
    return synth.make_inputs(wl, device, weights)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits(t)
    return t.detach().cpu().numpy()


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def max_rel_err(got_bits: np.ndarray, ref_bits: np.ndarray) -> float:
    g, r = bf16_f64(got_bits), bf16_f64(ref_bits)
    assert np.all(np.isfinite(g)), "non-finite values in the GPU output"
    scale = np.abs(r).max()
    return float(np.abs(g - r).max() / (scale if scale > 0 else 1.0))


def assert_close(got_bits, ref_bits, tol=REL_TOL, what="output"):
    e = max_rel_err(got_bits, ref_bits)
    assert e <= tol, f"{what}: max|d|/max|ref| = {e:.3e} > {tol}"
    return e


def assert_gates(gpu_gate: np.ndarray, ref_gate: np.ndarray):
    np.testing.assert_allclose(gpu_gate, ref_gate, rtol=1e-6, atol=1e-30)
