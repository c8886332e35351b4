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


def assert_combine_close(got_bits, ref_bits, what="output"):
    """Element-wise bound for a combine of the same bf16 rows with the same gates:
    the two sides accumulate in fp32 in the same order but may round the products
    differently (fused multiply-add against multiply then add), which can move the
    final bf16 rounding by at most one bf16 ulp, i.e. |gpu - ref| <= 2^-7 |ref|."""
    g, r = bf16_f64(got_bits), bf16_f64(ref_bits)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values in the GPU output"
    bad = np.abs(g - r) > np.abs(r) * 2.0 ** -7 + 1e-30
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond one bf16 ulp, e.g. " \
        f"{g[bad][:3]} vs {r[bad][:3]}"


def band_covering_tokens(offsets, perm, wl, n_random=48, band_rows=128, seed=None):
    """Tokens to check through the oracle's definition path: for every 128-row band
    of every expert (rows [offsets[e] + 128 i, ...)), the token of one seeded random
    row of it; plus the first and last tokens and n_random seeded random tokens."""
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    toks = [0, wl.T - 1]
    for e in range(len(offsets) - 1):
        for r0 in range(int(offsets[e]), int(offsets[e + 1]), band_rows):
            r1 = min(r0 + band_rows, int(offsets[e + 1]))
            toks.append(int(perm[rng.integers(r0, r1)]) // wl.k)
    toks.extend(rng.choice(wl.T, size=min(n_random, wl.T), replace=False).tolist())
    return np.unique(np.asarray(toks, np.int64)).astype(np.int32)


def bands_covered(offsets, perm, wl, toks, band_rows=128) -> bool:
    """Does every band hold a routed row of one of the tokens?"""
    tset = set(int(t) for t in toks)
    for e in range(len(offsets) - 1):
        for r0 in range(int(offsets[e]), int(offsets[e + 1]), band_rows):
            r1 = min(r0 + band_rows, int(offsets[e + 1]))
            if not any(int(p) // wl.k in tset for p in perm[r0:r1]):
                return False
    return True
