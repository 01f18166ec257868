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

The exchanges use NCCL's all-to-all (the plain transport; a kernel that
stores rows straight into the owner's memory over NVLink, overlapped with
the copies, is the next step and is not built here).  With no process
group (one GPU) the exchanges are the identity and the path reduces to the
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


def dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
             num_experts: int, pg=None) -> Dispatched:
    """Multi-GPU dispatch of this rank's tokens (x [T, H] bf16, topk_idx
    [T, k], topk_weights [T, k] fp32, all on this rank's GPU), on the current
    stream (the one the collectives are ordered with)."""
    world, rank = _world(pg)
    E = num_experts
    lay = epx.layout(topk_idx, E, world)
    send = epx.dispatch(x, lay)
    meta_idx, meta_w = epx.route_meta(topk_idx, topk_weights, lay)
    counts = exchange_counts(lay.cnt_r, pg)          # synchronises the stream
    plan = send_plan(counts, rank)
    n = plan["n_send"]
    recv_x = exchange_rows(send[:n], plan, pg)
    recv_idx = exchange_rows(meta_idx[:n], plan, pg)
    recv_w = exchange_rows(meta_w[:n], plan, pg)
    lay_in = epx.layout(recv_idx, E, world)
    _, expanded = epx.dispatch_expand(recv_x, lay_in, expand_only=True)
    return Dispatched(lay, plan, recv_x, recv_idx, recv_w, lay_in, expanded, pg)


def combine(h: Dispatched, expert_out: torch.Tensor, residual: torch.Tensor = None,
            partial_dtype=torch.float32) -> torch.Tensor:
    """Multi-GPU combine: expert_out holds the expert outputs of h.expanded's
    rows.  The local reduce leaves one partial row per received row, in
    receive order; those travel back by the reversed plan and land in the
    source's receive layout, where the epilogue sums each token's partials
    (plus `residual`, if given) and rounds once to bf16."""
    part = epx.combine_local_reduce(expert_out, h.recv_w, h.layout_in,
                                    partial_dtype=partial_dtype)
    back = exchange_rows(part[:h.plan["n_recv"]], h.plan, h.pg, reverse=True)
    return epx.combine_epilogue(back, h.layout, residual=residual)
