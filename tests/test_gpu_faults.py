"""Failure detection without a GPU fault: the debug flag makes the producer never
publish that the first row band's GEMM1 tiles are stored, so the GEMM2 tile that
reads those rows waits until its bound runs out; the kernel records
MOE_ERR_TIMEOUT in the status block and returns (every other wait ends early),
and the next call on the same context and workspace succeeds and is correct."""
import numpy as np
import pytest
import torch

from combine_overlap_b200 import synth
import gpu_util as gu

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("combine_overlap_b200.moe")


def test_consumer_timeout_is_reported_and_recoverable():
    wl = synth.small("fault", 300, 256, 128, 4, 2)
    inp = gu.inputs(wl)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
    args = (inp["x"], inp["logits"], inp["W1"], inp["W3"], inp["W2"], wl.k, ws)
    good = moe.layer_forward(*args, mode=moe.MODE_SEQUENTIAL).clone()
    assert moe.get_status(ws)[0] == moe.MOE_OK
    for mode in (moe.MODE_OVERLAPPED, moe.MODE_SEQUENTIAL):
        moe.layer_forward(*args, mode=mode, flags=moe.DBG_SKIP_FLAG_BAND, timeout_us=20000)
        code, _, _ = moe.get_status(ws)
        assert code == moe.MOE_ERR_TIMEOUT, mode
    again = moe.layer_forward(*args, mode=moe.MODE_OVERLAPPED)
    assert moe.get_status(ws)[0] == moe.MOE_OK
    assert torch.equal(again, good)
