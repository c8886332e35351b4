"""The whole layer, steps (a)-(e), on the GPU.

* Small layers, every element: GPU vs the oracle within 2e-2 * max|ref|; routing
  outputs bit-exact (including layers whose tokens fill 3, 1 or none of the
  consumer's staging slots), for both the CTA-pair and the single-CTA tile
  variants; the overlapped mode bit-identical to the sequential mode
  for every consumer-SM count tried (cost model, 1, 2, 4, 8, 32), segment size
  mgb in {1, 2, 3} and with or without producers joining the combine.
* Every benchmark workload at full size (the Mixtral-shaped, fine-grained and
  imbalanced layers and all twelve T x router layers of the d=4096/E=32 grid), in
  the configuration the benchmark times: routing outputs in full; a sample of
  tokens through the oracle's token-by-token definition path that holds at least
  one routed row of every 128-row band (so every producer tile row group and
  every consumer band is checked), plus the first and last tokens and a seeded
  random set; overlapped == sequential in full.  The same at full size for the
  other tile variants and the schedule options (side combine warps, the two
  GEMM1 gathers, the interleaved queue, evict-first stores) on a few layers each,
  the schedule options also bit-identical to the default in full.
* The same layers with identity experts (MOE_DBG_IDENTITY_EXPERTS): route,
  permute and combine, checked element by element over the whole output.
* The oracle's fp32-intermediate variant (h kept in fp32): the GPU output is
  within the same bound of it as of the bf16-h oracle."""
import os

import numpy as np
import pytest
import torch

from combine_overlap_b200 import synth
import gpu_util as gu

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")

SMALL = [
    synth.WORKLOADS["tiny"],
    synth.small("ragged_T", 333, 256, 256, 5, 2, "zipf"),
    synth.small("k3_multi_band", 600, 512, 384, 4, 3),
    synth.small("hot_expert", 500, 256, 128, 16, 4, "hot"),
    synth.small("one_token", 1, 256, 128, 8, 2),
    # consumer staging regimes: k*d*2 bytes per token against 192 KB of slots
    synth.small("three_slots", 300, 4096, 128, 16, 8, "normal2"),    # 64 KB -> 3 slots < 5 warps
    synth.small("one_slot", 200, 12288, 128, 8, 8),                  # 192 KB -> 1 slot
    synth.small("no_slot", 160, 12544, 128, 8, 8),                   # 196 KB -> register fallback
]


def _forward(inp, wl, ws, mode, **kw):
    out, extra = moe.layer_forward(inp["x"], inp["logits"], inp["W1"], inp["W3"], inp["W2"], wl.k,
                                   ws, mode, outputs=True, **kw)
    code, c, nb = moe.get_status(ws)
    assert code == moe.MOE_OK, moe.status_string(code)
    return out, extra, c


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_layer_small(orc, wl):
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    ref = orc.forward(gu.host(inp["x"]), gu.host(inp["logits"]), gu.host(inp["W1"]),
                      gu.host(inp["W3"]), gu.host(inp["W2"]), wl.k)
    pair = moe.SCHED_CTA_PAIR
    if wl.name == "tiny":
        # the fp32-intermediate reading of the oracle (h not rounded to bf16)
        ref32 = orc.forward(gu.host(inp["x"]), gu.host(inp["logits"]), gu.host(inp["W1"]),
                            gu.host(inp["W3"]), gu.host(inp["W2"]), wl.k, fp32_h=True)
        dflt32, _, _ = _forward(inp, wl, ws, moe.MODE_OVERLAPPED)
        gu.assert_close(gu.host(dflt32), ref32["out"], what="tiny vs fp32-h oracle")
        # identity experts: route, permute and combine alone, every element
        refI = orc.forward(gu.host(inp["x"]), gu.host(inp["logits"]), None, None, None, wl.k,
                           identity=True)
        for mode in (moe.MODE_SEQUENTIAL, moe.MODE_OVERLAPPED):
            outI, _, _ = _forward(inp, wl, ws, mode, flags=moe.DBG_IDENTITY_EXPERTS)
            gu.assert_combine_close(gu.host(outI), refI["out"], what=f"tiny identity experts {mode}")
    seq, extra, _ = _forward(inp, wl, ws, moe.MODE_SEQUENTIAL, flags=pair)
    # the sequential mode combines after the FFN only: no token combined in-kernel
    assert moe.debug_tokens_combined(ws, wl.T, wl.d, wl.f, wl.E, wl.k) == 0
    assert np.array_equal(gu.host(extra["topk_idx"]), ref["topk_idx"])
    gu.assert_gates(gu.host(extra["topk_gate"]), ref["topk_gate"])
    assert np.array_equal(gu.host(extra["counts"]), ref["counts"])
    assert np.array_equal(gu.host(extra["offsets"]), ref["offsets"])
    assert np.array_equal(gu.host(extra["perm"]), ref["perm"])
    gu.assert_close(gu.host(seq), ref["out"], what=f"sequential ({wl.name})")
    seq_bits = gu.host(seq)
    for kw in (dict(), dict(consumer_sms=1), dict(consumer_sms=2), dict(consumer_sms=4),
               dict(consumer_sms=8), dict(consumer_sms=32), dict(mgb=2), dict(mgb=3, consumer_sms=3),
               dict(flags=moe.SCHED_NO_JOIN, consumer_sms=2)):
        ovl, _, c = _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=pair | kw.pop("flags", 0), **kw)
        assert c >= 2 and c % 2 == 0      # whole CTA pairs, at least one
        assert np.array_equal(gu.host(ovl), seq_bits), f"overlapped {kw} differs from sequential"
    # the single-CTA (128-row tile) variant: same checks
    one = moe.SCHED_ONE_CTA
    seq1, _, _ = _forward(inp, wl, ws, moe.MODE_SEQUENTIAL, flags=one)
    gu.assert_close(gu.host(seq1), ref["out"], what=f"sequential, one CTA ({wl.name})")
    for kw in (dict(), dict(consumer_sms=1), dict(consumer_sms=5, mgb=2)):
        ovl1, _, c = _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=one | kw.pop("flags", 0), **kw)
        assert np.array_equal(gu.host(ovl1), gu.host(seq1)), f"one-CTA overlapped {kw} differs"
    # 256-row tiles on single CTAs: per band the same MMA shape and K order as the
    # 128-row tiles, so the same bits, in both modes
    wide = moe.SCHED_WIDE_CTA
    for mode, kw in ((moe.MODE_SEQUENTIAL, dict()), (moe.MODE_OVERLAPPED, dict()),
                     (moe.MODE_OVERLAPPED, dict(consumer_sms=3, mgb=2))):
        out3, _, _ = _forward(inp, wl, ws, mode, flags=wide, **kw)
        assert np.array_equal(gu.host(out3), gu.host(seq1)), f"wide-CTA tiles {mode} {kw} differ"
    # the default picks single-CTA tiles of 256 rows (T*k/E >= 256) or 128 rows:
    # either way the bits of the 128-row variant
    dflt, _, _ = _forward(inp, wl, ws, moe.MODE_OVERLAPPED)
    assert moe.tile_variant(wl.T, wl.f, wl.E, wl.k) == (3 if wl.T * wl.k >= 256 * wl.E else 1)
    assert np.array_equal(gu.host(dflt), gu.host(seq1))
    # GEMM1 reading its A rows from x instead of x_perm -- copied by extra warps
    # with cp.async, or by TMA gather4: same arithmetic on the same rows, so the
    # same bits, in every tile variant;
    # and single CTAs loading the weight tiles one 64-column atom per copy (3-D
    # maps) instead of one 4-D copy per operand: the same bytes in the same places
    # and CTA pairs running an expert's odd last band as a full 256-row tile
    # and the schedule and store-policy variants: GEMM2 tiles interleaved with
    # GEMM1 tiles (instead of all GEMM1 tiles first), evict-first h/y stores
    for fl in (moe.SCHED_GATHER_LSU | one, moe.SCHED_GATHER_LSU | wide,
               moe.SCHED_GATHER_LSU | wide | moe.SCHED_INTERLEAVE,
               moe.SCHED_GATHER_A | pair, moe.SCHED_GATHER_A | one, moe.SCHED_GATHER_A | wide,
               moe.SCHED_GATHER_A | wide | moe.SCHED_B_PER_ATOM, moe.SCHED_B_PER_ATOM | one,
               moe.SCHED_B_PER_ATOM | wide,
               moe.SCHED_FULL_TILES | pair, moe.SCHED_INTERLEAVE | one, moe.SCHED_INTERLEAVE | pair,
               moe.SCHED_INTERLEAVE | wide, moe.SCHED_EVICT_FIRST | wide,
               moe.SCHED_EVICT_FIRST | moe.SCHED_INTERLEAVE | one):
        gat, _, _ = _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=fl)
        base = seq_bits if fl & pair else gu.host(seq1)
        assert np.array_equal(gu.host(gat), base), f"flags {fl:#x} differ"
    # side combine warps: the producers' CTAs do the arrivals and combine ready
    # tokens while the tiles run (no dedicated consumer unless asked for), with
    # or without joining, interleaved or not; CTA pairs ignore the flag.  Same bits.
    side = moe.SCHED_SIDE_COMBINE
    for fl, kw in ((side | one, dict()), (side | wide, dict()), (side, dict()),
                   (side | wide | moe.SCHED_INTERLEAVE, dict()), (side | one | moe.SCHED_INTERLEAVE, dict()),
                   (side | wide, dict(consumer_sms=2)), (side | one | moe.SCHED_NO_JOIN, dict()),
                   (side | wide | moe.SCHED_NO_JOIN | moe.SCHED_INTERLEAVE, dict(consumer_sms=3)),
                   (side | wide, dict(mgb=2)), (side | pair, dict())):
        sd, _, c = _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=fl, **kw)
        assert 0 <= moe.debug_tokens_combined(ws, wl.T, wl.d, wl.f, wl.E, wl.k) <= wl.T
        base = seq_bits if fl & pair else gu.host(seq1)
        assert np.array_equal(gu.host(sd), base), f"side combine flags {fl:#x} {kw} differ"
        if not fl & pair:
            assert c == kw.get("consumer_sms", 0)
    # SiLU in its exp form (the default uses the hardware tanh): other bits in h,
    # the same bound against the oracle, and the same bits in every mode and tile
    # variant
    exp_bits = None
    for fl in (moe.SCHED_EXP_SILU | one, moe.SCHED_EXP_SILU | wide,
               moe.SCHED_EXP_SILU | wide | moe.SCHED_INTERLEAVE):
        for mode in (moe.MODE_SEQUENTIAL, moe.MODE_OVERLAPPED):
            out_e, _, _ = _forward(inp, wl, ws, mode, flags=fl)
            gu.assert_close(gu.host(out_e), ref["out"], what=f"exp silu {fl:#x} ({wl.name})")
            exp_bits = gu.host(out_e) if exp_bits is None else exp_bits
            assert np.array_equal(gu.host(out_e), exp_bits), f"exp silu {fl:#x} mode {mode} differs"


def test_layer_repeat_bitwise():
    wl = synth.small("repeat", 700, 512, 256, 8, 2, "zipf")
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    first = moe.layer_forward(inp["x"], inp["logits"], inp["W1"], inp["W3"], inp["W2"], wl.k, ws)
    first = first.clone()
    for _ in range(20):
        again = moe.layer_forward(inp["x"], inp["logits"], inp["W1"], inp["W3"], inp["W2"], wl.k, ws)
        assert torch.equal(again, first)


FULL = ["mixtral", "fine_grained", "imbalanced"] + \
    [f"sweep_T{T}_{r}" for T in (512, 2048, 8192, 32768) for r in ("uniform", "zipf", "hot")]
# (workload, flags): every layer in its default variant (256-row single-CTA
# tiles from 256 rows per expert up, 128-row tiles below), and the other variants
# on a few
FULL_CASES = [(n, 0) for n in FULL] + [("mixtral", 0x4), ("mixtral", 0x20), ("fine_grained", 0x20),
                                        ("sweep_T512_hot", 0x100)] + \
    [(n, 0x1000) for n in ("mixtral", "fine_grained", "imbalanced", "sweep_T2048_uniform",
                           "sweep_T32768_uniform", "sweep_T512_zipf")] + \
    [(n, 0x8000) for n in ("fine_grained", "sweep_T8192_zipf")] + \
    [(n, 0x10) for n in ("sweep_T2048_hot", "sweep_T512_uniform")] + \
    [(n, 0x400) for n in ("mixtral", "imbalanced")] + \
    [(n, 0x800) for n in ("fine_grained", "sweep_T32768_hot")]
_FLAG_IDS = {0: "default", 0x4: "one", 0x20: "pair", 0x100: "wide", 0x1000: "side", 0x8000: "lsu_gather",
             0x10: "tma_gather", 0x400: "interleave", 0x800: "evict_first"}


@pytest.mark.parametrize("name,flags", FULL_CASES, ids=[f"{n}-{_FLAG_IDS[f]}" for n, f in FULL_CASES])
def test_layer_full_size_sampled(orc, name, flags):
    assert flags in (0, moe.SCHED_ONE_CTA, moe.SCHED_CTA_PAIR, moe.SCHED_WIDE_CTA, moe.SCHED_SIDE_COMBINE,
                     moe.SCHED_GATHER_LSU, moe.SCHED_GATHER_A, moe.SCHED_INTERLEAVE, moe.SCHED_EVICT_FIRST)
    wl = synth.WORKLOADS[name]
    orc.set_threads(os.cpu_count() or 1)
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    ovl, extra, c = _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=flags)
    ovl_bits = gu.host(ovl)
    seq, _, _ = _forward(inp, wl, ws, moe.MODE_SEQUENTIAL, flags=flags)
    assert np.array_equal(gu.host(seq), ovl_bits), "overlapped differs from sequential"
    if flags in (moe.SCHED_SIDE_COMBINE, moe.SCHED_GATHER_LSU, moe.SCHED_GATHER_A, moe.SCHED_INTERLEAVE,
                 moe.SCHED_EVICT_FIRST):
        # a schedule option changes where and when, not what: the default's bits
        dflt, _, _ = _forward(inp, wl, ws, moe.MODE_OVERLAPPED)
        assert np.array_equal(gu.host(dflt), ovl_bits), f"flags {flags:#x} differ from the default"
    # routing in full
    oidx, ogate = orc.route(gu.host(inp["logits"]), wl.k)
    assert np.array_equal(gu.host(extra["topk_idx"]), oidx)
    gu.assert_gates(gu.host(extra["topk_gate"]), ogate)
    oc, oo, op, _ = orc.permute(oidx, wl.E)
    assert np.array_equal(gu.host(extra["counts"]), oc)
    assert np.array_equal(gu.host(extra["offsets"]), oo)
    assert np.array_equal(gu.host(extra["perm"]), op)
    # sampled tokens through the definition path: one routed row of every band,
    # the first and last tokens, and a seeded random set
    toks = gu.band_covering_tokens(oo, op, wl, n_random=48 if wl.d * wl.f * wl.k > 4096 * 4096 * 4 else 96)
    assert gu.bands_covered(oo, op, wl, toks)
    ref = orc.tokens(gu.host(inp["x"]), oidx, ogate, gu.host(inp["W1"]), gu.host(inp["W3"]),
                     gu.host(inp["W2"]), toks)
    gu.assert_close(ovl_bits[toks], ref, what=f"{name} sampled tokens ({len(toks)})")
    if name == "mixtral" and flags == 0:
        # the fp32-intermediate reading of the oracle: within the same bound
        ref32 = orc.tokens(gu.host(inp["x"]), oidx, ogate, gu.host(inp["W1"]), gu.host(inp["W3"]),
                           gu.host(inp["W2"]), toks, fp32_h=True)
        gu.assert_close(ovl_bits[toks], ref32, what=f"{name} sampled tokens vs fp32-h oracle")


@pytest.mark.parametrize("name", ["fine_grained", "imbalanced", "sweep_T32768_zipf", "sweep_T512_hot"])
def test_layer_full_size_identity_experts(orc, name):
    """Identity experts: the whole output of route -> permute -> combine at full
    size against the oracle's, element by element, in both modes."""
    wl = synth.WORKLOADS[name]
    orc.set_threads(os.cpu_count() or 1)
    inp = gu.inputs(wl, weights=False)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    ref = orc.forward(gu.host(inp["x"]), gu.host(inp["logits"]), None, None, None, wl.k, identity=True)
    for mode in (moe.MODE_SEQUENTIAL, moe.MODE_OVERLAPPED):
        out, extra = moe.layer_forward(inp["x"], inp["logits"], None, None, None, wl.k, ws, mode,
                                       outputs=True, flags=moe.DBG_IDENTITY_EXPERTS, d_ff=wl.f)
        assert moe.get_status(ws)[0] == moe.MOE_OK
        assert np.array_equal(gu.host(extra["perm"]), ref["perm"])
        gu.assert_combine_close(gu.host(out), ref["out"], what=f"{name} identity experts, mode {mode}")


def _check_variants(orc, wl, inp):
    """Every tile variant against the oracle, and overlapped == sequential in each."""
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    ref = orc.forward(gu.host(inp["x"]), gu.host(inp["logits"]), gu.host(inp["W1"]),
                      gu.host(inp["W3"]), gu.host(inp["W2"]), wl.k)
    for fl in (moe.SCHED_ONE_CTA, moe.SCHED_CTA_PAIR, moe.SCHED_WIDE_CTA):
        seq, extra, _ = _forward(inp, wl, ws, moe.MODE_SEQUENTIAL, flags=fl)
        assert np.array_equal(gu.host(extra["topk_idx"]), ref["topk_idx"])
        assert np.array_equal(gu.host(extra["counts"]), ref["counts"])
        assert np.array_equal(gu.host(extra["perm"]), ref["perm"])
        gu.assert_close(gu.host(seq), ref["out"], what=f"{wl.name} flags {fl:#x}")
        for kw in (dict(), dict(consumer_sms=4)):
            ovl, _, _ = _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=fl, **kw)
            assert np.array_equal(gu.host(ovl), gu.host(seq)), (fl, kw)


def test_layer_max_experts(orc):
    # the largest expert count and top-k the library accepts: E = 256, k = 8, so
    # about 9 rows per expert and hundreds of one-band groups (pairs: half tiles)
    wl = synth.small("max_experts", 300, 256, 128, 256, 8, "normal2")
    _check_variants(orc, wl, gu.inputs(wl))


@pytest.mark.parametrize("k", [1, 2])
def test_layer_every_token_one_expert(orc, k):
    # every token's first choice is expert 3 (its logit raised by 50): one expert
    # holds T rows in 8 bands (k = 1 leaves the other 7 experts empty)
    wl = synth.small(f"one_expert_k{k}", 1000, 256, 256, 8, k)
    inp = gu.inputs(wl)
    inp["logits"][:, 3] += 50.0
    _check_variants(orc, wl, inp)


def test_gather_variants_refused():
    # the cp.async gather warps exist for single-CTA tiles only
    wl = synth.WORKLOADS["tiny"]
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    with pytest.raises(moe.MoEError) as e:
        _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=moe.SCHED_GATHER_LSU | moe.SCHED_CTA_PAIR)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
    # ... and the side combine warps are the same extra warps: not both
    with pytest.raises(moe.MoEError) as e:
        _forward(inp, wl, ws, moe.MODE_OVERLAPPED, flags=moe.SCHED_GATHER_LSU | moe.SCHED_SIDE_COMBINE)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED


def test_binding_rejects_mismatched_shapes():
    # the library sees pointers only; the binding refuses shapes that would make it
    # read or write out of bounds, before anything is launched
    wl = synth.WORKLOADS["tiny"]
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    x, logits, W1, W3, W2 = (inp[n] for n in ("x", "logits", "W1", "W3", "W2"))
    with pytest.raises(ValueError):      # W2 given as [E][d][f]
        moe.layer_forward(x, logits, W1, W3, W1, wl.k, ws)
    with pytest.raises(ValueError):      # logits for another expert count
        moe.layer_forward(x, logits[:, :wl.E - 1].contiguous(), W1, W3, W2, wl.k, ws)
    with pytest.raises(ValueError):      # output rows short
        moe.layer_forward(x, logits, W1, W3, W2, wl.k, ws, out=x[:-1].clone())
    with pytest.raises(ValueError):      # combine: gates for more tokens than y rows
        moe.combine(x, torch.zeros(wl.T, dtype=torch.int32, device="cuda"),
                    torch.zeros((wl.T, wl.k), dtype=torch.float32, device="cuda"))
