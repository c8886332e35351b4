"""Seeded random layer shapes inside the documented preconditions (T >= 1,
1 <= k <= min(E, 8), E <= 256, d % 256 == 0, f % 128 == 0), each checked element
by element against the oracle, with routing bit-exact and the overlapped mode
(cost model and a fixed split) bit-identical to the sequential mode."""
import numpy as np
import pytest

from combine_overlap_b200 import synth
import gpu_util as gu

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")


def _shapes(n=10, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.choice([1, 2, 3, 5, 8, 13, 32, 64]))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.choice([1, 7, 33, 129, 255, 400, 777]))
        d = int(rng.choice([256, 512, 768]))
        f = int(rng.choice([128, 256, 384, 640]))
        router = str(rng.choice(["uniform", "zipf", "hot", "normal2"]))
        out.append(synth.small(f"fz{i}_T{T}_d{d}_f{f}_E{E}_k{k}_{router}", T, d, f, E, k, router,
                               int(rng.integers(1, 1 << 30))))
    return out


@pytest.mark.parametrize("wl", _shapes(), ids=lambda w: w.name)
def test_fuzz_layer(orc, wl):
    wl = synth.Workload(wl.name, wl.T, wl.d, wl.f, wl.E, wl.k, wl.router, wl.seed, 1.0, 0.05)
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    ref = orc.forward(gu.host(inp["x"]), gu.host(inp["logits"]), gu.host(inp["W1"]),
                      gu.host(inp["W3"]), gu.host(inp["W2"]), wl.k)
    args = (inp["x"], inp["logits"], inp["W1"], inp["W3"], inp["W2"], wl.k, ws)
    seq, extra = moe.layer_forward(*args, mode=moe.MODE_SEQUENTIAL, outputs=True)
    assert moe.get_status(ws)[0] == moe.MOE_OK
    assert np.array_equal(gu.host(extra["topk_idx"]), ref["topk_idx"])
    assert np.array_equal(gu.host(extra["perm"]), ref["perm"])
    gu.assert_close(gu.host(seq), ref["out"], what=wl.name)
    for kw in (dict(), dict(consumer_sms=6, mgb=2)):
        ovl = moe.layer_forward(*args, mode=moe.MODE_OVERLAPPED, **kw)
        assert moe.get_status(ws)[0] == moe.MOE_OK
        assert np.array_equal(gu.host(ovl), gu.host(seq)), kw
