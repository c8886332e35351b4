"""Steps (a) route and (b) permute on the GPU against the oracle: top-k ids,
counts, offsets, the permutation, its inverse and the permuted rows bit for
bit; gates within 1e-6 relative.  Covers every benchmark workload at full size
(routing is cheap) plus edge cases: one token, ragged token counts across the
128-token blocks, one expert, k = E, exact ties, 256 experts, a hot expert."""
import numpy as np
import pytest
import torch

from combine_overlap_b200 import synth
import gpu_util as gu

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")

FULL = ["tiny", "mixtral", "fine_grained", "imbalanced", "sweep_T512_uniform",
        "sweep_T8192_zipf", "sweep_T32768_hot"]
EDGE = [
    synth.small("one_token", 1, 256, 128, 4, 2),
    synth.small("ragged", 1000, 256, 128, 6, 3, "zipf"),
    synth.small("one_expert", 130, 256, 128, 1, 1),
    synth.small("k_eq_E", 257, 256, 128, 8, 8),
    synth.small("many_experts", 515, 256, 128, 256, 8, "normal2"),
    synth.small("hot", 777, 256, 128, 16, 2, "hot"),
]


def _ties(T=300, E=12):
    g = torch.Generator().manual_seed(5)
    return torch.randint(-2, 3, (T, E), generator=g).to(torch.float32)


def _check_route(orc, logits_dev, k):
    T, E = logits_dev.shape
    ws = moe.alloc_workspace(T, 256, 128, E, k)
    idx, gate, cnt = moe.route(logits_dev, k, ws, counts=True)
    torch.cuda.synchronize()
    oidx, ogate = orc.route(gu.host(logits_dev), k)
    assert np.array_equal(gu.host(idx), oidx)
    gu.assert_gates(gu.host(gate), ogate)
    assert np.array_equal(gu.host(cnt), np.bincount(oidx.reshape(-1), minlength=E))
    return idx


def _check_permute(orc, x_dev, idx_dev, E):
    T, k = idx_dev.shape
    ws = moe.alloc_workspace(T, 256, 128, E, k)
    counts, offsets, perm, row_of, x_perm = moe.permute(x_dev, idx_dev, E, ws)
    torch.cuda.synchronize()
    oc, oo, op, orow = orc.permute(gu.host(idx_dev), E)
    assert np.array_equal(gu.host(counts), oc)
    assert np.array_equal(gu.host(offsets), oo)
    assert np.array_equal(gu.host(perm), op)
    assert np.array_equal(gu.host(row_of), orow)
    assert np.array_equal(gu.host(x_perm), orc.gather(gu.host(x_dev), op, k))


@pytest.mark.parametrize("name", FULL)
def test_route_permute_workloads(orc, name):
    wl = synth.WORKLOADS[name]
    inp = gu.inputs(wl, weights=False)
    idx = _check_route(orc, inp["logits"], wl.k)
    _check_permute(orc, inp["x"], idx, wl.E)


@pytest.mark.parametrize("wl", EDGE, ids=lambda w: w.name)
def test_route_permute_edges(orc, wl):
    inp = gu.inputs(wl, weights=False)
    idx = _check_route(orc, inp["logits"], wl.k)
    _check_permute(orc, inp["x"], idx, wl.E)


@pytest.mark.parametrize("k", [1, 2, 5, 8])
def test_route_ties(orc, k):
    logits = _ties().cuda()
    _check_route(orc, logits, k)


def test_route_repeatable():
    wl = synth.WORKLOADS["fine_grained"]
    logits = synth.make_logits(wl, "cuda")
    ws = moe.alloc_workspace(wl.T, 256, 128, wl.E, wl.k)
    a = moe.route(logits, wl.k, ws)
    b = moe.route(logits, wl.k, ws)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
