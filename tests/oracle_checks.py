"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check takes an ``oracle.Oracle`` handle and raises AssertionError on a
mismatch.  They are run on the oracle (all must pass) and on builds with a
planted mistake (each mistake must fail at least one), see
test_oracle_pins.py and test_oracle_mutants.py.

What pins what (definitions: "Fine-grained Computation-Communication Overlap
via Tile-level Signaling and Scheduling for Mixture-of-Experts", Section 2.1
and Section 3.2.1):
  route    -- brute force over all k-subsets (the defining property of top-k
              with ties to the lower id); k = E equals the library softmax;
              the two-expert logistic closed form; sum of gates = 1; adding an
              exactly representable constant to a row changes nothing.
  permute  -- numpy's stable argsort; bijection and segment invariants.
  experts  -- E = 1, k = 1 is a dense SwiGLU FFN: numpy float64 matmuls within
              bf16 error; W1 = W3 = 0 gives exactly 0; W2 * 2 gives exactly 2*out;
              identity experts give bf16(sum_j g_j x_t).
  layer    -- the hand-worked example in tests/golden; the token-by-token
              definition path equals the permuted path bit for bit; permuting
              tokens permutes outputs; relabelling experts changes nothing.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np
import scipy.special
import torch

from combine_overlap_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bf16_bits_of(a: np.ndarray) -> np.ndarray:
    return synth.bf16_bits(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def small_layer(T=24, d=32, f=48, E=5, k=2, seed=7, router="uniform", w_std=0.25):
    wl = synth.small("pin", T, d, f, E, k, router, seed)
    wl = synth.Workload(wl.name, T, d, f, E, k, router, seed, 1.0, w_std)
    inp = synth.make_inputs(wl)
    return dict(x=synth.bf16_bits(inp["x"]), logits=inp["logits"].numpy(),
                W1=synth.bf16_bits(inp["W1"]), W3=synth.bf16_bits(inp["W3"]),
                W2=synth.bf16_bits(inp["W2"]), k=k)


# ---------------------------------------------------------------- route ----

def check_route_bruteforce(o):
    rng = np.random.default_rng(11)
    for E in (3, 4, 6):
        for k in range(1, E + 1):
            # integer logits in a narrow range -> many exact ties
            logits = rng.integers(-2, 3, size=(40, E)).astype(np.float32)
            logits[0] = 0.0               # all tied
            logits[1, :] = -0.0           # signed zeros tie too
            logits[1, 0] = 0.0
            idx, gate = o.route(logits, k)
            for t in range(logits.shape[0]):
                l = logits[t]

                def beats(a, b):
                    return l[a] > l[b] or (l[a] == l[b] and a < b)

                winners = [S for S in itertools.combinations(range(E), k)
                           if all(beats(a, b) for a in S for b in range(E) if b not in S)]
                assert len(winners) == 1, (E, k, t)
                S = winners[0]
                # slot j of expert e = number of chosen experts that beat e
                slot = {e: sum(beats(o2, e) for o2 in S) for e in S}
                expect = [None] * k
                for e, j in slot.items():
                    expect[j] = e
                assert list(idx[t]) == expect, (E, k, t, list(idx[t]), expect)


def check_route_softmax(o):
    rng = np.random.default_rng(12)
    E = 8
    logits = rng.normal(size=(64, E)).astype(np.float32)
    idx, gate = o.route(logits, E)                    # k = E: full softmax
    full = scipy.special.softmax(logits.astype(np.float64), axis=1)
    ref = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(gate, ref, rtol=2e-7, atol=0)
    np.testing.assert_allclose(gate.astype(np.float64).sum(1), 1.0, rtol=0, atol=1e-6)
    # two selected experts: logistic closed form g0 = 1 / (1 + exp(l1 - l0))
    idx2, gate2 = o.route(logits, 2)
    l0 = np.take_along_axis(logits, idx2[:, :1].astype(np.int64), 1)[:, 0].astype(np.float64)
    l1 = np.take_along_axis(logits, idx2[:, 1:].astype(np.int64), 1)[:, 0].astype(np.float64)
    np.testing.assert_allclose(gate2[:, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=2e-7)
    np.testing.assert_allclose(gate2[:, 1], 1.0 / (1.0 + np.exp(l0 - l1)), rtol=2e-7)
    # descending order of the selected logits
    sel = np.take_along_axis(logits, idx.astype(np.int64), 1)
    assert np.all(np.diff(sel, axis=1) <= 0)


def check_route_shift(o):
    rng = np.random.default_rng(13)
    logits = rng.integers(-4, 5, size=(50, 7)).astype(np.float32)
    for k in (1, 2, 3, 7):
        i1, g1 = o.route(logits, k)
        i2, g2 = o.route(logits + np.float32(2.0), k)
        assert np.array_equal(i1, i2)
        assert np.array_equal(g1.view(np.uint32), g2.view(np.uint32))


# -------------------------------------------------------------- permute ----

def check_permute(o):
    rng = np.random.default_rng(14)
    for (T, E, k) in ((1, 1, 1), (37, 5, 2), (64, 8, 3), (200, 16, 6)):
        logits = rng.normal(size=(T, E)).astype(np.float32)
        logits[:, 0] += 3.0 * (E > 2)          # a hot expert; leaves others empty-ish
        idx, _ = o.route(logits, k)
        counts, offsets, perm, row_of = o.permute(idx, E)
        flat = idx.reshape(-1)
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
        assert offsets[-1] == T * k
        ref = np.argsort(flat, kind="stable")
        assert np.array_equal(perm, ref)
        assert np.array_equal(np.sort(perm), np.arange(T * k))
        assert np.array_equal(row_of[perm], np.arange(T * k))
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


# -------------------------------------------------------------- experts ----

def _dense_ref(x, W1, W3, W2):
    x = bf16_to_f64(x)
    W1, W3, W2 = (bf16_to_f64(w) for w in (W1, W3, W2))
    a, b = x @ W1, x @ W3
    h = a / (1.0 + np.exp(-a)) * b
    return h @ W2


def check_dense_ffn(o):
    for (T, d, f) in ((16, 24, 40), (9, 64, 16)):
        L = small_layer(T=T, d=d, f=f, E=1, k=1, seed=21)
        res = o.forward(L["x"], L["logits"], L["W1"], L["W3"], L["W2"], 1)
        assert np.all(res["topk_gate"] == 1.0)
        ref = _dense_ref(L["x"], L["W1"][0], L["W3"][0], L["W2"][0])
        got = bf16_to_f64(res["out"])
        tol = 1.5e-2 * np.abs(ref).max()
        assert np.abs(got - ref).max() <= tol, (np.abs(got - ref).max(), tol)
        # also row by row through the single-row entry point
        for t in range(T):
            y = o.ffn_row(L["x"][t], L["W1"][0], L["W3"][0], L["W2"][0])
            assert np.array_equal(y, res["out"][t])


def check_ffn_special(o):
    L = small_layer(seed=22)
    base = o.forward(L["x"], L["logits"], L["W1"], L["W3"], L["W2"], L["k"])
    zero = np.zeros_like(L["W1"])
    z = o.forward(L["x"], L["logits"], zero, zero, L["W2"], L["k"])
    assert np.all(bf16_to_f64(z["out"]) == 0.0)
    W2x2 = bf16_bits_of(2.0 * bf16_to_f64(L["W2"]))
    dbl = o.forward(L["x"], L["logits"], L["W1"], L["W3"], W2x2, L["k"])
    assert np.array_equal(bf16_to_f64(dbl["out"]), 2.0 * bf16_to_f64(base["out"]))
    # fp32-intermediate variant stays within bf16 error of the bf16 one
    f32 = o.forward(L["x"], L["logits"], L["W1"], L["W3"], L["W2"], L["k"], fp32_h=True)
    ref = bf16_to_f64(f32["out"])
    assert np.abs(bf16_to_f64(base["out"]) - ref).max() <= 2e-2 * np.abs(ref).max()


def check_identity_experts(o):
    L = small_layer(T=40, d=16, E=6, k=3, seed=23)
    res = o.forward(L["x"], L["logits"], None, None, None, L["k"], identity=True)
    g = res["topk_gate"].astype(np.float64)
    x = bf16_to_f64(L["x"])
    ref = g.sum(1, keepdims=True) * x             # sum_j g_j x_t, exact in f64
    got = bf16_to_f64(res["out"])
    # one bf16 rounding of an fp32 sum of k terms
    assert np.all(np.abs(got - ref) <= np.abs(ref) * (2.0 ** -8 + 1e-6) + 1e-30)
    assert np.abs(got - x).max() <= 2.0 ** -7 * np.abs(x).max()


# ---------------------------------------------------------------- layer ----

def check_golden(o):
    with open(os.path.join(GOLDEN, "tiny_handworked.json")) as fh:
        g = json.load(fh)
    ex = g["expected"]
    x = bf16_bits_of(np.array(g["x"]))
    W1, W3, W2 = (bf16_bits_of(np.array(g[n])) for n in ("W1", "W3", "W2"))
    logits = np.array(g["logits"], np.float32)
    res = o.forward(x, logits, W1, W3, W2, g["k"])
    assert res["topk_idx"].tolist() == ex["topk_idx"]
    assert res["topk_gate"].tolist() == ex["topk_gate"]
    assert res["counts"].tolist() == ex["counts"]
    assert res["offsets"].tolist() == ex["offsets"]
    assert res["perm"].tolist() == ex["perm"]
    counts, offsets, perm, row_of = o.permute(res["topk_idx"], g["E"])
    assert row_of.tolist() == ex["row_of"]
    xp = o.gather(x, perm, g["k"])
    y = o.expert_ffn(xp, offsets, W1, W3, W2)
    assert bf16_to_f64(y).tolist() == ex["y_by_row"]
    assert bf16_to_f64(res["out"]).tolist() == ex["out"]


def check_definition_path(o):
    for (T, d, f, E, k, router) in ((30, 32, 48, 5, 2, "uniform"), (17, 16, 24, 8, 3, "zipf"),
                                    (12, 8, 8, 4, 4, "hot")):
        L = small_layer(T=T, d=d, f=f, E=E, k=k, seed=24, router=router)
        res = o.forward(L["x"], L["logits"], L["W1"], L["W3"], L["W2"], k)
        toks = np.arange(T, dtype=np.int32)
        alt = o.tokens(L["x"], res["topk_idx"], res["topk_gate"], L["W1"], L["W3"], L["W2"], toks)
        assert np.array_equal(alt, res["out"])
        # the step-by-step entry points compose to the same layer
        counts, offsets, perm, row_of = o.permute(res["topk_idx"], E)
        xp = o.gather(L["x"], perm, k)
        y = o.expert_ffn(xp, offsets, L["W1"], L["W3"], L["W2"])
        out = o.combine(y, row_of, res["topk_gate"])
        assert np.array_equal(out, res["out"])


def check_token_permutation(o):
    L = small_layer(T=33, seed=25)
    res = o.forward(L["x"], L["logits"], L["W1"], L["W3"], L["W2"], L["k"])
    pi = np.random.default_rng(3).permutation(33)
    res2 = o.forward(L["x"][pi], L["logits"][pi], L["W1"], L["W3"], L["W2"], L["k"])
    assert np.array_equal(res2["out"], res["out"][pi])


def check_expert_relabel(o):
    L = small_layer(T=29, E=6, k=3, seed=26)
    res = o.forward(L["x"], L["logits"], L["W1"], L["W3"], L["W2"], L["k"])
    sigma = np.random.default_rng(4).permutation(6)      # new column c holds old expert sigma[c]
    res2 = o.forward(L["x"], L["logits"][:, sigma], L["W1"][sigma], L["W3"][sigma],
                     L["W2"][sigma], L["k"])
    assert np.array_equal(res2["out"], res["out"])
    assert np.array_equal(sigma[res2["topk_idx"]], res["topk_idx"])


ALL_CHECKS = [
    check_route_bruteforce, check_route_softmax, check_route_shift, check_permute,
    check_dense_ffn, check_ffn_special, check_identity_experts, check_golden,
    check_definition_path, check_token_permutation, check_expert_relabel,
]
