"""moe_layer_forward inside a CUDA graph: the call is asynchronous and allocates
nothing, so a caller can capture it once and replay it; every replay re-runs
routing, planning and the persistent kernel on whatever the input buffers hold.
Replays with new inputs must give exactly the eager result for those inputs."""
import pytest
import torch

from combine_overlap_b200 import synth

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")


@pytest.mark.parametrize("mode", ["overlapped", "sequential"])
def test_layer_in_cuda_graph(mode):
    m = moe.MODE_OVERLAPPED if mode == "overlapped" else moe.MODE_SEQUENTIAL
    wl = synth.small("graph", 700, 512, 256, 8, 2, "zipf", 31)
    inp = synth.make_inputs(wl, "cuda")
    x = inp["x"].clone()
    logits = inp["logits"].clone()
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    out = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    args = lambda: (x, logits, inp["W1"], inp["W3"], inp["W2"], wl.k, ws)
    moe.layer_forward(*args(), mode=m, out=out)            # eager warm-up (sets up the device)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.layer_forward(*args(), mode=m, out=out)
    for seed in (101, 202):
        other = synth.Workload("graph", wl.T, wl.d, wl.f, wl.E, wl.k, wl.router, seed)
        x.copy_(synth.make_x(other, "cuda"))
        logits.copy_(synth.make_logits(other, "cuda"))
        g.replay()
        torch.cuda.synchronize()
        assert moe.get_status(ws)[0] == moe.MOE_OK
        replayed = out.clone()
        ref = moe.layer_forward(*args(), mode=m)
        torch.cuda.synchronize()
        assert torch.equal(replayed, ref)
