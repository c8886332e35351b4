"""Expert-parallel exchange plumbing (combine_overlap_b200/ep.py) on CPU gloo
ranks.  Each rank routes, permutes and gathers its own tokens, dispatches its
routed rows to the experts' owners, each owner computes its experts' FFN on what
it received, the results come back to their home ranks, and each home combines.
The oracle stands in for the device compute on both sides.  The result must be
bit-identical to the oracle's whole layer on the rank's tokens with every expert
local: the exchange moves rows and never changes their arithmetic."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from combine_overlap_b200 import ep, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _as_i16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16))


def _worker(rank, world, port, E, router, out):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o = oracle.get()
        o.set_threads(1)
        T = 40 + 13 * rank                        # ragged shards
        d, f, k = 128, 64, 2
        wl = synth.Workload("ep", T, d, f, E, k, router, 1000 + rank, 1.0, 0.05)
        inp = synth.make_inputs(wl, "cpu")
        # the same weights on every rank (the tests' stand-in for each owner's share)
        wts = synth.make_inputs(synth.Workload("ep_w", 1, d, f, E, k, router, 77, 1.0, 0.05), "cpu")
        x = synth.bf16_bits(inp["x"])
        logits = inp["logits"].numpy()
        W = [synth.bf16_bits(wts[n]) for n in ("W1", "W3", "W2")]

        # home: route, permute, gather (one GPU's steps (a) and (b))
        idx, gate = o.route(logits, k)
        counts, offsets, perm, row_of = o.permute(idx, E)
        x_perm = o.gather(x, perm, k)

        # exchange: counts, then the routed rows to their owners
        ex = ep.plan_exchange(torch.from_numpy(counts.astype(np.int64)), world)
        assert sum(ex.send_rows) == T * k
        recv = ep.dispatch(_as_i16(x_perm), ex)
        order, offs = ep.owner_order(ex)
        assert sorted(order.tolist()) == list(range(sum(ex.recv_rows)))

        # owner: its experts' FFN on the received rows, grouped by local expert
        el = ep.local_experts(E, world)
        lo = rank * el
        x_own = recv[order].numpy().view(np.uint16)
        Wl = [w[lo:lo + el] for w in W]
        y_own = o.expert_ffn(x_own, offs.numpy().astype(np.int32), *Wl)

        # back home, in the order the rows left; then the combine as on one GPU
        y_home = ep.return_rows(_as_i16(y_own), order, ex).numpy().view(np.uint16)
        got = o.combine(y_home, row_of, gate)
        ref = o.forward(x, logits, *W, k)["out"]
        out[rank] = dict(equal=bool(np.array_equal(got, ref)),
                         recv=sum(ex.recv_rows), sent=ex.send_rows)
    finally:
        dist.destroy_process_group()


# "hot" sends most rows to expert 0; with 16 experts over 2 ranks, Zipf routing
# leaves some (source, expert) runs empty
@pytest.mark.parametrize("world,E,router", [(2, 8, "uniform"), (2, 8, "hot"), (4, 8, "zipf"),
                                            (2, 16, "zipf")])
def test_ep_exchange_matches_whole_layer(world, E, router):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, E, router, out), nprocs=world,
                       start_method="spawn", join=True)
    total_sent = sum(sum(out[r]["sent"]) for r in range(world))
    assert total_sent == sum(out[r]["recv"] for r in range(world))
    for r in range(world):
        assert out[r]["equal"], f"rank {r}: expert-parallel result differs from the whole layer"


def test_owner_order_groups_by_expert():
    # two sources, three local experts; source-major received rows
    c = torch.tensor([[2, 0, 1], [1, 3, 0]], dtype=torch.int64)
    ex = ep.Exchange(send_rows=[0, 0], recv_rows=c.sum(1).tolist(), recv_counts=c)
    order, offs = ep.owner_order(ex)
    # received rows: s0 = [e0, e0, e2], s1 = [e0, e1, e1, e1]
    assert order.tolist() == [0, 1, 3, 4, 5, 6, 2]
    assert offs.tolist() == [0, 3, 6, 7]
    with pytest.raises(ValueError):
        ep.local_experts(10, 4)
    assert ep.owner_of(5, 8, 4) == 2
