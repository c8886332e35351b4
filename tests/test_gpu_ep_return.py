"""The fused expert-parallel return on W virtual ranks of one GPU
(moe_ep_owner_forward + moe_ep_home_combine, driven by ep.virtual_ranks_forward).

Each owner's consumer CTAs store every finished row band into its home rank's
return buffer and bump the home's per-token arrival words; each home combines.
The rows are computed by the same kernels with the same K order as on one GPU,
and the home combine is moe_combine's arithmetic, so every rank's output must be
bit-identical to moe_layer_forward on that rank's tokens with all experts local
-- for 2 and 4 ranks, uniform, Zipf and hot routing, both owner modes, dedicated
return CTAs or not, and merged middle segments (mgb).  The arrival words must be
back at zero afterwards.  A home whose rows never arrive reports MOE_ERR_TIMEOUT
(a bounded wait on a word nothing writes) and the context stays usable."""
import pytest
import torch

from combine_overlap_b200 import ep, synth
import gpu_util as gu

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")


def _ranks(W, T0, d, f, E, k, router, seed):
    xs, ls = [], []
    for r in range(W):
        wl = synth.Workload(f"ep{r}", T0 + 37 * r, d, f, E, k, router, seed + 11 * r)
        xs.append(synth.make_x(wl, "cuda"))
        ls.append(synth.make_logits(wl, "cuda"))
    W1, W3, W2 = synth.make_weights(synth.Workload("epw", 1, d, f, E, k, router, seed + 999), "cuda")
    return xs, ls, W1, W3, W2


def _reference(xs, ls, W1, W3, W2, k):
    E, d, f = W1.shape
    refs = []
    for x, l in zip(xs, ls):
        ws = moe.alloc_workspace(x.shape[0], d, f, E, k)
        refs.append(moe.layer_forward(x, l, W1, W3, W2, k, ws, moe.MODE_SEQUENTIAL).clone())
        assert moe.get_status(ws)[0] == moe.MOE_OK
    return refs


def _check(outs, state, refs, what):
    for r, (o, ref) in enumerate(zip(outs, refs)):
        assert int(state["status"][r].item()) == 0, f"{what}: home {r} status"
        assert torch.equal(o, ref), f"{what}: rank {r} differs from the one-GPU layer"
        assert int(state["homes"][r]["arrive"].abs().sum().item()) == 0, f"{what}: arrival words not reset"
    for o, own in enumerate(state["owners"]):
        if own["N"] > 0:
            assert moe.get_status(own["ws"])[0] == moe.MOE_OK, f"{what}: owner {o}"


@pytest.mark.parametrize("W", [2, 4])
@pytest.mark.parametrize("router", ["uniform", "zipf", "hot"])
def test_ep_return_matches_one_gpu_layer(W, router):
    k = 2 if W == 2 else 3
    xs, ls, W1, W3, W2 = _ranks(W, 300, 512, 256, 8, k, router, 4242)
    refs = _reference(xs, ls, W1, W3, W2, k)
    cases = [dict(mode=moe.MODE_OVERLAPPED), dict(mode=moe.MODE_SEQUENTIAL),
             dict(mode=moe.MODE_OVERLAPPED, consumer_sms=2),
             dict(mode=moe.MODE_OVERLAPPED, consumer_sms=3, mgb=2),
             dict(mode=moe.MODE_OVERLAPPED, flags=moe.SCHED_ONE_CTA),
             dict(mode=moe.MODE_OVERLAPPED, flags=moe.SCHED_INTERLEAVE, consumer_sms=1)]
    for kw in cases:
        outs, state = ep.virtual_ranks_forward(xs, ls, W1, W3, W2, k, **kw)
        torch.cuda.synchronize()
        _check(outs, state, refs, f"W={W} {router} {kw}")


def test_ep_return_benchmark_shape():
    # 4 ranks of the d=4096 / E=32 / top-4 layer, 2048 tokens each (8 local experts
    # per owner, ~256 rows per (expert, source) segment: 256-row tiles, many bands)
    W, k = 4, 4
    xs, ls, W1, W3, W2 = _ranks(W, 2048, 4096, 2048, 32, k, "zipf", 777)
    refs = _reference(xs, ls, W1, W3, W2, k)
    for kw in (dict(mode=moe.MODE_OVERLAPPED), dict(mode=moe.MODE_OVERLAPPED, consumer_sms=4, mgb=2),
               dict(mode=moe.MODE_SEQUENTIAL)):
        outs, state = ep.virtual_ranks_forward(xs, ls, W1, W3, W2, k, **kw)
        torch.cuda.synchronize()
        _check(outs, state, refs, f"benchmark shape {kw}")


def test_ep_owner_plan_is_remote_first():
    # the owner's band table: remote bands (home != owner) all come before local ones
    W, k, E = 4, 2, 8
    xs, ls, W1, W3, W2 = _ranks(W, 700, 256, 128, E, k, "uniform", 99)
    outs, state = ep.virtual_ranks_forward(xs, ls, W1, W3, W2, k)
    torch.cuda.synchronize()
    for o, own in enumerate(state["owners"]):
        nb = moe.get_status(own["ws"])[2]
        dests = moe.ep_band_dest(own["ws"], own["N"], 256, 128, E // W, W, nb)
        ranks = [int(r) for r, _ in dests]
        first_local = ranks.index(o) if o in ranks else len(ranks)
        assert all(r != o for r in ranks[:first_local]) and all(r == o for r in ranks[first_local:]), \
            f"owner {o}: band destinations {ranks}"


def test_ep_home_times_out_when_nothing_arrives():
    # no owner runs: every arrival word stays 0, so the home's bounded wait runs out
    T, d, k = 64, 256, 2
    y = torch.zeros((T * k, d), dtype=torch.bfloat16, device="cuda")
    arrive = torch.zeros(T, dtype=torch.int32, device="cuda")
    row_of = torch.arange(T * k, dtype=torch.int32, device="cuda")
    gate = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    _, st = moe.ep_home_combine(y, arrive, row_of, gate, timeout_us=2000)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_ERR_TIMEOUT
    # the context is fine: with the arrivals in place the same call completes
    arrive.fill_(k)
    out, st = moe.ep_home_combine(y, arrive, row_of, gate, timeout_us=2000)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(arrive.abs().sum().item()) == 0
    assert torch.equal(out, torch.zeros_like(out))
