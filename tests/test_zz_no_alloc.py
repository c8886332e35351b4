"""moe_permute_noalloc, the permutation for callers that cannot allocate device
memory (a pooled runtime, a plug-in host, code that must not call cudaMalloc
where it permutes): called through the C ABI, it must give exactly what
moe_permute gives with a caller workspace, on two calls in a row with different
inputs -- the second call reuses the fixed scratch array the first one left
behind.  Kept in its own file, collected last."""
import pytest
import torch

from combine_overlap_b200 import synth

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")


def _case(wl):
    x = synth.make_x(wl, "cuda")
    logits = synth.make_logits(wl, "cuda")
    ws = moe.alloc_workspace(wl.T, 256, 128, wl.E, wl.k)
    idx, _ = moe.route(logits, wl.k, ws)
    return x, idx, ws


def test_permute_noalloc_matches_permute_twice():
    assert moe._lib.moe_permute_noalloc_scratch_bytes() >= 1 << 20
    cases = [synth.WORKLOADS["fine_grained"], synth.small("second", 3001, 512, 128, 40, 3, "hot", 99)]
    for wl in cases:
        x, idx, ws = _case(wl)
        ref = moe.permute(x, idx, wl.E, ws)
        got = moe.permute_noalloc(x, idx, wl.E)
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm", "row_of", "x_perm"), got, ref):
            assert torch.equal(a, b), f"{wl.name}: {name} differs from moe_permute"


def test_permute_noalloc_rejects_oversize():
    x = torch.zeros((65537, 256), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((65537, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.permute_noalloc(x, idx, 4)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
