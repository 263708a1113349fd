"""Expert-parallel exchange of the dispatch rows between ranks.

The AWS Neuron "Permute A2AV Kernel API Reference" (permute_a2av, return
values) packs the [C, H] send buffer destination-major and returns a [4, EP]
uint32 table -- send counts, send displacements, receive counts, receive
displacements, all in elements -- for the all_to_all_v that ships it; the
Mojo MAX ep_comm dispatch and combine kernels move the same rows to the
ranks that own the experts and back.

Here one process drives one GPU and the S segments of the layout are the S
ranks of the expert-parallel group: segment s (experts [sL, (s+1)L)) of the
dispatch output is the block of rows for rank s.  The steps, in the order
every rank takes them:

  exchange_counts         all-to-all of meta row 0; writes the receive counts
                          and displacements into meta rows 2 and 3
  exchange_expert_counts  each source rank's row count for every local expert
  dispatch_exchange       the payload rows (bf16 rows, FP8 / FP4 code rows or
                          their scale rows: any row width) to their expert's rank
  combine_exchange        the expert outputs back along the reverse route, to
                          the rows the dispatch output had, ready for moe_combine

In packed mode a segment's rows are contiguous (meta row 1 is the exclusive
cumsum), so the split of a send buffer is meta row 0 / H rows per rank; in
capacity mode ([E, Ce, H], static positions) every segment is its full
L * Ce rows, padding included.  The collectives are torch.distributed
all_to_all_single calls (NCCL over NVLink / NVSwitch on GPUs, gloo on CPU);
the split sizes are read to the host once per exchange_counts.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Route:
    """Rows this rank sends to and receives from every rank of the group."""
    send_rows: list[int]
    recv_rows: list[int]

    @property
    def recv_total(self) -> int:
        return sum(self.recv_rows)

    @property
    def send_total(self) -> int:
        return sum(self.send_rows)


def _world(group) -> int:
    return dist.get_world_size(group)


def _u32(row: torch.Tensor) -> torch.Tensor:
    # meta holds uint32 bit patterns in an int32 tensor
    return row.to(torch.int64) & 0xFFFFFFFF


def _to_u32_bits(v: torch.Tensor) -> torch.Tensor:
    # int64 values in [0, 2^32) -> the same bits in an int32 tensor
    return torch.where(v >= 2 ** 31, v - 2 ** 32, v).to(torch.int32)


def exchange_counts(meta: torch.Tensor, hidden: int, num_experts: int,
                    expert_capacity: int = 0, group=None) -> Route:
    """All-to-all of the send counts (meta row 0, elements).  Fills meta rows
    2 and 3 with the receive counts and their exclusive cumsum (elements),
    as the [4, EP] table of permute_a2av, and returns the row route."""
    S = meta.shape[1]
    if S != _world(group):
        raise ValueError(f"meta has {S} segments for a group of {_world(group)} ranks")
    if expert_capacity > 0:
        seg = (num_experts // S) * expert_capacity
        send_rows = [seg] * S
        send_elems = torch.full((S,), seg * hidden, dtype=torch.int64, device=meta.device)
    else:
        send_elems = _u32(meta[0]).contiguous()
        send_rows = [int(v) // hidden for v in send_elems.tolist()]
    recv_elems = torch.empty_like(send_elems)
    dist.all_to_all_single(recv_elems, send_elems, group=group)
    displs = torch.cumsum(recv_elems, 0) - recv_elems
    meta[2].copy_(_to_u32_bits(recv_elems))
    meta[3].copy_(_to_u32_bits(displs))
    return Route(send_rows=send_rows, recv_rows=[int(v) // hidden for v in recv_elems.tolist()])


def exchange_expert_counts(expert_counts: torch.Tensor, group=None) -> torch.Tensor:
    """[S, L] int32: row s holds the rows source rank s routed to each of this
    rank's L experts (its expert_counts[rank*L : (rank+1)*L])."""
    S = _world(group)
    E = expert_counts.numel()
    send = expert_counts.to(torch.int32).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.view(S, E // S)


def _row_bytes(t: torch.Tensor) -> torch.Tensor:
    # rows as raw bytes [rows, bytes per row]: one collective for any dtype
    return t.contiguous().view(torch.uint8).reshape(t.shape[0], -1)


def dispatch_exchange(rows: torch.Tensor, route: Route, group=None) -> torch.Tensor:
    """Ship segment s of `rows` (the dispatch output, or its code or scale
    rows) to rank s; returns the received rows, source rank by source rank."""
    if rows.shape[0] < route.send_total:
        raise ValueError("fewer rows than the route sends")
    send = _row_bytes(rows[:route.send_total])
    out = torch.empty((route.recv_total, send.shape[1]), dtype=torch.uint8, device=rows.device)
    dist.all_to_all_single(out, send, output_split_sizes=route.recv_rows,
                           input_split_sizes=route.send_rows, group=group)
    return out.view(rows.dtype).reshape((route.recv_total,) + tuple(rows.shape[1:]))


def combine_exchange(expert_rows: torch.Tensor, route: Route, out: torch.Tensor | None = None,
                     group=None) -> torch.Tensor:
    """Return the expert outputs of the received rows to their source ranks:
    row i of segment s comes back to row i of segment s of the dispatch
    output it left, so moe_combine can use the layout's pair_slot as is.
    Rows past the route (packed-mode padding) are left as they are in `out`
    (zero-filled when `out` is not given)."""
    if expert_rows.shape[0] != route.recv_total:
        raise ValueError("expert rows do not match the route")
    if out is None:
        out = torch.zeros((route.send_total,) + tuple(expert_rows.shape[1:]),
                          dtype=expert_rows.dtype, device=expert_rows.device)
    send = _row_bytes(expert_rows)
    back = torch.empty((route.send_total, send.shape[1]), dtype=torch.uint8,
                       device=expert_rows.device)
    dist.all_to_all_single(back, send, output_split_sizes=route.send_rows,
                           input_split_sizes=route.recv_rows, group=group)
    out[:route.send_total].copy_(
        back.view(expert_rows.dtype).reshape((route.send_total,) + tuple(expert_rows.shape[1:])))
    return out
