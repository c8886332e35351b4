"""Steps (c1)+(c2), the grouped SwiGLU expert FFN on tcgen05, against the oracle
on the same permuted rows: y within 2e-2 * max|ref|.  Shapes span several
row bands per expert, ragged last bands, near-empty and empty experts, a single
row, and several column tiles of both GEMMs -- each in every tile variant:
128-row tiles on single CTAs, 256-row tiles on CTA pairs (with half tiles) and
256-row tiles on single CTAs."""
import numpy as np
import pytest
import torch

from combine_overlap_b200 import synth
import gpu_util as gu

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")

CASES = [
    synth.small("single_row", 1, 256, 128, 4, 1),
    synth.small("one_band", 64, 256, 128, 4, 2),
    synth.small("ragged", 300, 512, 256, 6, 2, "zipf"),
    synth.small("multi_band", 700, 256, 384, 3, 3),
    synth.small("empty_experts", 200, 256, 256, 32, 2, "zipf"),
    synth.WORKLOADS["tiny"],
    synth.small("many_bands", 1100, 256, 256, 4, 2, "zipf"),   # several full pair groups per expert
]

VARIANTS = {"one_cta": moe.SCHED_ONE_CTA, "cta_pair": moe.SCHED_CTA_PAIR, "wide_cta": moe.SCHED_WIDE_CTA}


def _run(orc, wl, w_std=0.02, flags=0):
    wl = synth.Workload(wl.name, wl.T, wl.d, wl.f, wl.E, wl.k, wl.router, wl.seed, 1.0, w_std)
    inp = gu.inputs(wl)
    oidx, _ = orc.route(gu.host(inp["logits"]), wl.k)
    counts, offsets, perm, row_of = orc.permute(oidx, wl.E)
    xp = orc.gather(gu.host(inp["x"]), perm, wl.k)
    R = wl.T * wl.k
    xp_dev = synth.from_bf16_bits(xp).cuda()
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    h, y = moe.grouped_ffn(xp_dev, torch.from_numpy(offsets).cuda(), inp["W1"], inp["W3"], inp["W2"],
                           wl.T, wl.k, ws, flags=flags)
    code, _, nb = moe.get_status(ws)
    assert code == moe.MOE_OK
    assert nb == int(sum((c + 127) // 128 for c in counts))
    yref = orc.expert_ffn(xp, offsets, gu.host(inp["W1"]), gu.host(inp["W3"]), gu.host(inp["W2"]))
    return gu.assert_close(gu.host(y)[:R], yref[:R], what=f"y ({wl.name})")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_grouped_ffn(orc, wl, variant):
    _run(orc, wl, flags=VARIANTS[variant])


@pytest.mark.parametrize("variant", VARIANTS)
def test_grouped_ffn_large_weights(orc, variant):
    # larger weights -> |a| of order 1-10, exercising the silu curve, not just its origin
    _run(orc, synth.small("wide_act", 300, 512, 256, 4, 2), w_std=0.1, flags=VARIANTS[variant])


def test_grouped_ffn_rejects_non_tile_flags():
    wl = synth.WORKLOADS["tiny"]
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    xp = torch.zeros((wl.T * wl.k, wl.d), dtype=torch.bfloat16, device="cuda")
    off = torch.zeros(wl.E + 1, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.grouped_ffn(xp, off, inp["W1"], inp["W3"], inp["W2"], wl.T, wl.k, ws,
                        flags=moe.SCHED_GATHER_A)
    assert e.value.code == moe.MOE_ERR_INVALID
