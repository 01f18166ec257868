"""Expert parallelism across GPUs: one rank per GPU, rank r owning experts
[r*E/R, (r+1)*E/R) -- the setting of the pages (DeepEP issue #48, question:
a token on rank 0 sent once to rank 1 for its experts M and N there; DeepEP
issue #760, Reproduction: a process group, dispatch returns a handle that
combine takes back).

Every step on the data runs in libepx's kernels; this module holds the
host-side plan and the two exchanges, which go through torch.distributed
(NCCL between GPUs; gloo on CPU for the host-logic tests):

  dispatch (source rank g)                     receiving rank r
  ------------------------                     ----------------
  ep_layout(topk_idx, E, R)  -> rank blocks
  ep_dispatch(x)             -> send rows, blocks of destination rank
  ep_route_meta(...)         -> per sent row: its routes kept on that rank
  all_gather(cnt_r)          -> counts[src, dst] on every rank
  all_to_all(rows, meta)     ----------------> recv_x, recv_idx, recv_w
                                               ep_layout(recv_idx, E, R)
                                               ep_dispatch_expand(expand only)
                                               (expert FFN on the expanded rows)
  combine                                      ep_combine_local_reduce ->
                                               one partial per received row
  all_to_all back (reverse plan) <------------
  ep_combine_epilogue(partials, layout) -> out

Received rows are ordered by source rank, then by the source's token order,
so rank r's received rows are exactly the rows a single GPU would put in
rank r's block of `recv` for the batches of all ranks concatenated in rank
order; the partials come back in each source's send order, which is the
receive layout of its own layout, so the epilogue of the two-stage combine
applies unchanged.

Two transports for the rows (`transport=`):
  "nccl" -- ep_dispatch into a send buffer, then NCCL's all-to-all (rows and
            their routing), and the same back for the partials;
  "p2p"  -- ep_dispatch_p2p stores every row and its routing straight into
            the receiving GPU's buffer (device pointers to the other ranks'
            buffers, mapped once through CUDA IPC by PeerBuffers), and
            ep_combine_local_reduce_p2p stores every partial row straight
            into its source's buffer; a one-word all-reduce on the stream
            after each kernel orders the ranks (no kernel waits on another
            GPU).  Placement and transfer are one kernel; there is no send
            buffer and no all-to-all.
Both give the same rows in the same places.  With no process group (one
GPU) the exchanges are the identity and the path reduces to the
single-GPU two-stage combine.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import epx


def _world(pg):
    if pg is None:
        return 1, 0
    import torch.distributed as dist
    return dist.get_world_size(pg), dist.get_rank(pg)


def send_plan(counts: torch.Tensor, rank: int) -> dict:
    """The all-to-all plan of one rank from counts[src, dst] (rows src sends
    to dst, gathered from every rank's layout cnt_r).

    send_splits[d]: rows this rank sends to rank d, in its send order (the
    layout's rank blocks, d ascending); recv_splits[s]: rows this rank
    receives from rank s, stored in s order; recv_offsets[s]: first received
    row from s.  The combine's return trip uses the same plan reversed."""
    c = counts.to(torch.int64).cpu()
    if c.dim() != 2 or c.shape[0] != c.shape[1] or not (0 <= rank < c.shape[0]):
        raise ValueError("counts must be [world, world] and rank inside it")
    if bool((c < 0).any()):
        raise ValueError("negative counts")
    send = [int(v) for v in c[rank, :]]
    recv = [int(v) for v in c[:, rank]]
    offs, run = [], 0
    for v in recv:
        offs.append(run)
        run += v
    return dict(send_splits=send, recv_splits=recv, recv_offsets=offs,
                n_send=sum(send), n_recv=run)


def p2p_plan(counts: torch.Tensor, rank: int) -> dict:
    """Where this rank's rows go under the peer-memory transport, from
    counts[src, dst] (rows src sends to dst).

    dispatch_row0[r]: first row of rank r's receive buffer that this rank
    writes (the rows r receives from lower ranks come first); back_first[s] /
    back_count[s]: the rows this rank received from source s ([first, first
    + count) of its receive order), whose partials go back to s at
    back_row0[s] = the first row of s's send block for this rank (s's blocks
    are in destination order).  n_recv / n_send: rows this rank receives /
    sends."""
    c = counts.to(torch.int64).cpu()
    if c.dim() != 2 or c.shape[0] != c.shape[1] or not (0 <= rank < c.shape[0]):
        raise ValueError("counts must be [world, world] and rank inside it")
    if bool((c < 0).any()):
        raise ValueError("negative counts")
    world = c.shape[0]
    dispatch_row0 = [int(c[:rank, r].sum()) for r in range(world)]
    back_first = [int(c[:s, rank].sum()) for s in range(world)]
    back_count = [int(c[s, rank]) for s in range(world)]
    back_row0 = [int(c[s, :rank].sum()) for s in range(world)]
    return dict(dispatch_row0=dispatch_row0, back_first=back_first, back_count=back_count,
                back_row0=back_row0, n_recv=int(c[:, rank].sum()), n_send=int(c[rank].sum()))


class PeerBuffers:
    """This rank's receive buffers (rows, routing) and partial-return buffer,
    and every other rank's, mapped into this process: the destinations of
    ep_dispatch_p2p and ep_combine_local_reduce_p2p.  Sized for batches of up
    to t_max tokens per rank: a rank receives at most one row per token of
    every rank (world * t_max rows) and gets back at most one partial per
    (token, rank) pair it sent (t_max * min(k, world) rows).  With one rank
    the buffers are plain local allocations."""

    def __init__(self, t_max: int, H: int, k: int, pg=None, partial_dtype=torch.float32,
                 device=None):
        world, rank = _world(pg)
        self.world, self.rank, self.pg = world, rank, pg
        self.H, self.k, self.partial_dtype = H, k, partial_dtype
        self.device = device if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.recv_cap = world * t_max
        self.back_cap = t_max * min(k, world)
        pbytes = 4 if partial_dtype == torch.float32 else 2
        shapes = [("rows", (self.recv_cap, H), torch.bfloat16, 2 * H),
                  ("meta_idx", (self.recv_cap, k), torch.int32, 4 * k),
                  ("meta_w", (self.recv_cap, k), torch.float32, 4 * k),
                  ("back", (self.back_cap, H), partial_dtype, pbytes * H)]
        self._own, self._opened = [], []
        self.local, self.peer = {}, {}
        # every rank's capacities (a peer's buffers are written up to its own)
        self.peer_recv_cap = [self.recv_cap] * world
        self.peer_back_cap = [self.back_cap] * world
        handles = {}
        for name, shape, dtype, row_bytes in shapes:
            nbytes = max(16, shape[0] * row_bytes)
            if world == 1:
                t = torch.empty(shape, dtype=dtype, device=self.device)
                self.local[name] = t
                self.peer[name] = [t]
                continue
            ptr, h = epx.ipc_malloc(nbytes)
            self._own.append(ptr)
            self.local[name] = epx.tensor_at(ptr, shape, dtype, self.device)
            handles[name] = (ptr, h)
        if world > 1:
            import torch.distributed as dist
            mine = dict(handles={n: h for n, (_, h) in handles.items()},
                        recv_cap=self.recv_cap, back_cap=self.back_cap, H=H, k=k,
                        partial=str(partial_dtype))
            gathered = [None] * world
            dist.all_gather_object(gathered, mine, group=pg)
            if any((g["H"], g["k"], g["partial"]) != (H, k, str(partial_dtype)) for g in gathered):
                self.close_local()
                raise ValueError("PeerBuffers: H, k and partial_dtype must agree on every rank")
            self.peer_recv_cap = [int(g["recv_cap"]) for g in gathered]
            self.peer_back_cap = [int(g["back_cap"]) for g in gathered]
            for name, _, _, _ in shapes:
                ptrs = []
                for r in range(world):
                    if r == rank:
                        ptrs.append(handles[name][0])
                    else:
                        p = epx.ipc_open(gathered[r]["handles"][name])
                        self._opened.append(p)
                        ptrs.append(p)
                self.peer[name] = ptrs

    def close_local(self):
        """Free this rank's own allocations (before any peer has mapped them)."""
        for p in self._own:
            epx.ipc_free(p)
        self._own = []

    def close(self):
        """Unmap the other ranks' buffers and free this rank's (collective:
        every rank calls it, so no peer still writes into freed memory)."""
        if self.world > 1:
            import torch.distributed as dist
            if self.device.type == "cuda":
                torch.cuda.synchronize(self.device)
            dist.barrier(group=self.pg)
        for p in self._opened:
            epx.ipc_close(p)
        for p in self._own:
            epx.ipc_free(p)
        self._opened, self._own = [], []


def _order_ranks(pg, device):
    """A one-word all-reduce on the current stream: every rank's kernels
    before it (its stores into other GPUs' buffers) have completed before any
    rank's work after it starts."""
    if pg is None:
        return
    import torch.distributed as dist
    dist.all_reduce(torch.zeros(1, dtype=torch.int32, device=device), group=pg)


def exchange_counts(cnt_r: torch.Tensor, pg=None) -> torch.Tensor:
    """counts[src, dst] from every rank's per-destination row counts
    (all-gather; the identity on one rank)."""
    world, _ = _world(pg)
    cnt = cnt_r.to(torch.int32).contiguous()
    if world == 1:
        return cnt.view(1, -1).cpu()
    import torch.distributed as dist
    if cnt.numel() != world:
        raise ValueError("one logical rank per process: R must equal the world size")
    parts = [torch.empty_like(cnt) for _ in range(world)]
    dist.all_gather(parts, cnt, group=pg)
    return torch.stack(parts).cpu()


def exchange_rows(rows: torch.Tensor, plan: dict, pg=None, reverse: bool = False) -> torch.Tensor:
    """Sends rows[...] by the plan (all-to-all with uneven splits): forward,
    send_splits out and recv_splits in; reverse, the other way round.  Rows
    of any dtype whose row size is a multiple of 4 bytes travel as int32
    words."""
    out_splits = plan["send_splits"] if reverse else plan["recv_splits"]
    in_splits = plan["recv_splits"] if reverse else plan["send_splits"]
    if rows.shape[0] != sum(in_splits):
        raise ValueError(f"{rows.shape[0]} rows for a plan sending {sum(in_splits)}")
    out = torch.empty((sum(out_splits),) + tuple(rows.shape[1:]), dtype=rows.dtype,
                      device=rows.device)
    world, _ = _world(pg)
    if world == 1:
        out.copy_(rows)
        return out
    row_bytes = rows[0].numel() * rows.element_size() if rows.dim() > 1 else rows.element_size()
    if row_bytes % 4:
        raise ValueError("row size must be a multiple of 4 bytes")
    import torch.distributed as dist
    words = row_bytes // 4
    dist.all_to_all_single(out.view(-1).view(torch.int32).view(-1, words),
                           rows.contiguous().view(-1).view(torch.int32).view(-1, words),
                           output_split_sizes=out_splits, input_split_sizes=in_splits,
                           group=pg)
    return out


@dataclass
class Dispatched:
    """Handle of one multi-GPU dispatch (what combine needs back)."""
    layout: epx.Layout          # this rank's tokens over all ranks
    plan: dict
    recv_x: torch.Tensor        # [n_recv, H] rows received from every rank
    recv_idx: torch.Tensor      # [n_recv, k] their routes kept on this rank
    recv_w: torch.Tensor        # [n_recv, k] their weights
    layout_in: epx.Layout       # layout of the received rows (all on this rank)
    expanded: torch.Tensor      # [n_recv*k, H] received rows once per local expert
    pg: object = None
    buffers: "PeerBuffers" = None   # peer-memory transport: where the partials go


def dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
             num_experts: int, pg=None, transport: str = "nccl",
             buffers: PeerBuffers = None) -> Dispatched:
    """Multi-GPU dispatch of this rank's tokens (x [T, H] bf16, topk_idx
    [T, k], topk_weights [T, k] fp32, all on this rank's GPU), on the current
    stream (the one the collectives are ordered with).  transport "p2p"
    needs `buffers` (PeerBuffers of this process group); the received rows
    are then views of buffers.local, valid until the next dispatch."""
    world, rank = _world(pg)
    E = num_experts
    if transport not in ("p2p", "nccl"):
        raise ValueError(f"unknown transport {transport!r}")
    if transport == "p2p":
        if buffers is None:
            raise ValueError("transport 'p2p' needs PeerBuffers")
        if buffers.world != world or buffers.rank != rank:
            raise ValueError("PeerBuffers belong to another process group")
        if x.shape[0] * world > buffers.recv_cap or x.shape[1] != buffers.H:
            raise ValueError("batch larger than the PeerBuffers were sized for")
    lay = epx.layout(topk_idx, E, world)
    if transport == "p2p":
        counts = exchange_counts(lay.cnt_r, pg)      # synchronises the stream
        plan = p2p_plan(counts, rank)
        plan.update(send_plan(counts, rank))
        if any(int(counts[:, r].sum()) > buffers.peer_recv_cap[r] for r in range(world)):
            raise ValueError("a rank receives more rows than its PeerBuffers hold")
        peers = [epx.PeerRows(buffers.peer["rows"][r], buffers.peer_recv_cap[r],
                              row0=plan["dispatch_row0"][r],
                              meta_idx=buffers.peer["meta_idx"][r],
                              meta_w=buffers.peer["meta_w"][r]) for r in range(world)]
        epx.dispatch_p2p(x, topk_idx, topk_weights, lay, peers)
        _order_ranks(pg, x.device)
        n = plan["n_recv"]
        recv_x = buffers.local["rows"][:n]
        recv_idx = buffers.local["meta_idx"][:n]
        recv_w = buffers.local["meta_w"][:n]
    elif transport == "nccl":
        send = epx.dispatch(x, lay)
        meta_idx, meta_w = epx.route_meta(topk_idx, topk_weights, lay)
        counts = exchange_counts(lay.cnt_r, pg)      # synchronises the stream
        plan = send_plan(counts, rank)
        n = plan["n_send"]
        recv_x = exchange_rows(send[:n], plan, pg)
        recv_idx = exchange_rows(meta_idx[:n], plan, pg)
        recv_w = exchange_rows(meta_w[:n], plan, pg)
    lay_in = epx.layout(recv_idx, E, world)
    _, expanded = epx.dispatch_expand(recv_x, lay_in, expand_only=True)
    return Dispatched(lay, plan, recv_x, recv_idx, recv_w, lay_in, expanded, pg,
                      buffers if transport == "p2p" else None)


def combine(h: Dispatched, expert_out: torch.Tensor, residual: torch.Tensor = None,
            partial_dtype=torch.float32) -> torch.Tensor:
    """Multi-GPU combine: expert_out holds the expert outputs of h.expanded's
    rows.  The local reduce leaves one partial row per received row, in
    receive order; those travel back (by the reversed plan, or stored
    straight into the sources' buffers) and land in the source's receive
    layout, where the epilogue sums each token's partials (plus `residual`,
    if given) and rounds once to bf16."""
    if h.buffers is not None:
        b = h.buffers
        if partial_dtype != b.partial_dtype:
            raise ValueError("partial_dtype differs from the PeerBuffers' one")
        world = b.world
        peers = [epx.PeerRows(b.peer["back"][s], b.peer_back_cap[s], row0=h.plan["back_row0"][s],
                              first=h.plan["back_first"][s], count=h.plan["back_count"][s])
                 for s in range(world)]
        epx.combine_local_reduce_p2p(expert_out, h.recv_w, h.layout_in, peers,
                                     partial_dtype=partial_dtype)
        _order_ranks(h.pg, expert_out.device)
        return epx.combine_epilogue(b.local["back"], h.layout, residual=residual)
    part = epx.combine_local_reduce(expert_out, h.recv_w, h.layout_in,
                                    partial_dtype=partial_dtype)
    back = exchange_rows(part[:h.plan["n_recv"]], h.plan, h.pg, reverse=True)
    return epx.combine_epilogue(back, h.layout, residual=residual)
