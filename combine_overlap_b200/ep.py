"""Expert parallelism across ranks: the host-side plumbing of the dispatch and
return exchanges.

W ranks; rank o owns the experts [o*E/W, (o+1)*E/W) ("Fine-grained
Computation-Communication Overlap via Tile-level Signaling and Scheduling for
Mixture-of-Experts", Section 2.1: each GPU hosts a subset of the experts;
Section 3.2.1: rows are laid out by owner).  Each rank routes and permutes its
own tokens with the library; the permutation groups its routed rows by expert,
so the rows bound for one owner are one contiguous run.  These functions turn
the permutation's offsets into exchange sizes, move the row runs with
torch.distributed all-to-all (NCCL on GPUs, gloo on CPUs), regroup an owner's
received rows by expert, and bring the results back to their home rank in the
order they left, where the combine runs as on one GPU.

This is the exchange with plain collectives, outside any kernel: the baseline
that a fused return (consumer SMs storing finished rows into the home rank's
buffer as each band completes) would replace.  Index bookkeeping only -- no
arithmetic of the layer happens here.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


def local_experts(E: int, W: int) -> int:
    """Experts per rank (E must be a multiple of W)."""
    if W < 1 or E % W != 0:
        raise ValueError(f"{E} experts do not split evenly over {W} ranks")
    return E // W


def owner_of(e: int, E: int, W: int) -> int:
    return e // local_experts(E, W)


@dataclass
class Exchange:
    """Sizes of one rank's dispatch and return, from both sides."""
    send_rows: list[int]          # [W] rows this rank sends to each owner
    recv_rows: list[int]          # [W] rows this rank receives from each source
    recv_counts: torch.Tensor     # [W][E/W] rows from each source for each local expert


def plan_exchange(counts: torch.Tensor, W: int, group=None) -> Exchange:
    """counts: [E] rows this rank routed to each expert (the permutation's
    counts).  Exchanges the per-expert counts with every rank (one all-to-all of
    E integers) and returns the split sizes of both exchanges."""
    E = counts.numel()
    el = local_experts(E, W)
    c = counts.to(torch.int64).reshape(W, el).contiguous()
    recv = torch.empty_like(c)
    dist.all_to_all_single(recv.view(-1), c.view(-1), group=group)
    return Exchange(send_rows=c.sum(1).tolist(), recv_rows=recv.sum(1).tolist(), recv_counts=recv)


def _exchange(rows: torch.Tensor, out_rows: int, out_split: list[int], in_split: list[int],
              group) -> torch.Tensor:
    """All-to-all of whole rows, moved as 32-bit words (the exchange only moves
    bits, and gloo has no 16-bit types).  Rows may be empty on either side."""
    tail = tuple(rows.shape[1:])
    row_bytes = rows.element_size()
    for n in tail:
        row_bytes *= n
    if row_bytes % 4 != 0:
        raise ValueError("row size must be a multiple of 4 bytes")
    words = row_bytes // 4
    if rows.shape[0] == 0:
        w = torch.empty((0, words), dtype=torch.int32, device=rows.device)
    else:
        w = rows.contiguous().view(torch.int32).reshape(rows.shape[0], words)
    out = w.new_empty((out_rows, words))
    dist.all_to_all_single(out, w, out_split, in_split, group=group)
    return out.view(rows.dtype).reshape((out_rows,) + tail)


def dispatch(rows: torch.Tensor, ex: Exchange, group=None) -> torch.Tensor:
    """rows: [R][...] this rank's routed rows in permutation order (expert
    ascending, so owner ascending).  Returns the rows this rank receives, source
    rank major, each source's rows in its own order (expert ascending)."""
    return _exchange(rows, sum(ex.recv_rows), ex.recv_rows, ex.send_rows, group)


def owner_order(ex: Exchange) -> tuple[torch.Tensor, torch.Tensor]:
    """For an owner's received rows (source major, expert ascending within each
    source): the order that groups them by local expert, sources ascending within
    an expert, and that grouping's offsets [E/W + 1].  order[i] is the received
    row placed at position i."""
    c = ex.recv_counts                                        # [W][el]
    W, el = c.shape
    src_start = torch.cumsum(c.sum(1), 0) - c.sum(1)          # first received row of each source
    within = torch.cumsum(c, 1) - c                           # first row of expert e inside source s
    parts = []
    for e in range(el):
        for s in range(W):
            n = int(c[s, e])
            if n:
                start = int(src_start[s] + within[s, e])
                parts.append(torch.arange(start, start + n, dtype=torch.int64))
    order = torch.cat(parts) if parts else torch.empty(0, dtype=torch.int64)
    per_expert = c.sum(0)
    offsets = torch.zeros(el + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(per_expert, 0)
    return order, offsets


def return_rows(rows_owner_order: torch.Tensor, order: torch.Tensor, ex: Exchange,
                group=None) -> torch.Tensor:
    """An owner's result rows, in owner_order, back to their home ranks.  Returns
    this rank's own routed rows' results in the order it dispatched them (its
    permutation order)."""
    received = torch.empty_like(rows_owner_order)
    received[order.to(rows_owner_order.device)] = rows_owner_order   # back to received order
    return _exchange(received, sum(ex.send_rows), ex.send_rows, ex.recv_rows, group)


def virtual_ranks_forward(xs, logits, W1, W3, W2, k: int, mode: int = 1, consumer_sms: int = 0,
                          mgb: int = 1, flags: int = 0, timeout_us: int = 0):
    """One expert-parallel MoE layer over W virtual ranks on the current GPU, with
    the fused return (Sections 3.2-3.3 of the paper).  xs[r], logits[r]: rank r's
    tokens and gate logits; W1, W3, W2: all E experts (rank o owns
    [o*E/W, (o+1)*E/W)).  Per rank: route and permute (the library); the dispatch
    all-to-all -- on several GPUs dispatch() above, over NCCL -- is stood in for by
    device copies of each home's row runs (with their home slots) into each
    owner's receive buffer; each owner runs moe_ep_owner_forward, whose consumer
    CTAs store every finished band into its home's return buffer and bump the
    home's arrival words; each home runs moe_ep_home_combine.  Returns (outs,
    state) with outs[r] rank r's layer output.  Owners run one after another, so
    no kernel here waits on a kernel that has not already finished."""
    from . import moe
    Wn = len(xs)
    E, d, f = W1.shape
    El = local_experts(E, Wn)
    dev = xs[0].device
    homes = []
    for r in range(Wn):
        T = xs[r].shape[0]
        ws = moe.alloc_workspace(T, d, f, E, k, dev)
        idx, gate = moe.route(logits[r], k, ws)
        counts, offsets, perm, row_of, x_perm = moe.permute(xs[r], idx, E, ws)
        homes.append(dict(T=T, ws=ws, idx=idx, gate=gate, counts=counts, offsets=offsets, perm=perm,
                          row_of=row_of, x_perm=x_perm,
                          y=torch.empty((T * k, d), dtype=torch.bfloat16, device=dev),
                          arrive=torch.zeros(T, dtype=torch.int32, device=dev)))
    offs = [h["offsets"].cpu() for h in homes]     # the exchange sizes, on the host
    owners = []
    for o in range(Wn):
        lo, hi = o * El, (o + 1) * El
        runs = [(int(offs[s][lo]), int(offs[s][hi])) for s in range(Wn)]
        x_recv = torch.cat([homes[s]["x_perm"][a:b] for s, (a, b) in enumerate(runs)])
        slot_recv = torch.cat([homes[s]["perm"][a:b] for s, (a, b) in enumerate(runs)])
        recv_counts = torch.stack([homes[s]["counts"][lo:hi] for s in range(Wn)]).contiguous()
        N = x_recv.shape[0]
        ws_o = torch.empty(moe.ep_owner_workspace_size(N, d, f, El, Wn), dtype=torch.uint8, device=dev)
        moe.ep_owner_forward(x_recv, slot_recv, recv_counts, W1[lo:hi], W3[lo:hi], W2[lo:hi], k, o,
                             [a for a, _ in runs], [h["y"] for h in homes], [h["arrive"] for h in homes],
                             ws_o, mode, consumer_sms=consumer_sms, mgb=mgb, flags=flags,
                             timeout_us=timeout_us)
        owners.append(dict(ws=ws_o, N=N, x_recv=x_recv, slot_recv=slot_recv, recv_counts=recv_counts))
    outs, statuses = [], []
    for h in homes:
        out, st = moe.ep_home_combine(h["y"], h["arrive"], h["row_of"], h["gate"], timeout_us=timeout_us)
        outs.append(out)
        statuses.append(st)
    return outs, dict(homes=homes, owners=owners, status=statuses)
