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

or, with the send fused into the permute (moe_permute_to_peers: each
segment's rows stored straight into the owning rank's receive buffer over
NVLink / NVSwitch), exchange_counts, then put_offsets (where this rank's
block starts in every receiver's buffer), the kernel, and a barrier before
the receivers read.

In packed mode a segment's rows are contiguous and start at meta row 1 / H
(the exclusive cumsum of the send counts); in capacity mode ([E, Ce, H],
static positions) segment s is its full L * Ce rows from s * L * Ce, padding
included.  The counts exchange is one all_to_all_single and the only step
that reads sizes to the host.  The payload steps are grouped point-to-point
transfers (torch.distributed batch_isend_irecv: on GPUs one NCCL group of
sends and receives over NVLink / NVSwitch, on CPU gloo): for every peer, one
send straight from the segment's first row (meta row 1) and one receive
straight into its block of the receive buffer (meta row 3), so no staging
copy of the send buffer is made; the segment a rank keeps is a local copy.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Route:
    """Rows this rank sends to and receives from every rank of the group,
    and where each segment starts: send_offsets in the dispatch output
    (meta row 1 / H), recv_offsets in the receive buffer (meta row 3 / H);
    both default to the exclusive cumsum of the row counts."""
    send_rows: list[int]
    recv_rows: list[int]
    send_offsets: list[int] | None = None
    recv_offsets: list[int] | None = None

    def __post_init__(self):
        def cumsum(rows):
            out, acc = [], 0
            for r in rows:
                out.append(acc)
                acc += r
            return out
        if self.send_offsets is None:
            self.send_offsets = cumsum(self.send_rows)
        if self.recv_offsets is None:
            self.recv_offsets = cumsum(self.recv_rows)

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
        send_offsets = [s * seg for s in range(S)]
        send_elems = torch.full((S,), seg * hidden, dtype=torch.int64, device=meta.device)
    else:
        send_elems = _u32(meta[0]).contiguous()
        send_rows = [int(v) // hidden for v in send_elems.tolist()]
        send_offsets = [int(v) // hidden for v in _u32(meta[1]).tolist()]
    recv_elems = torch.empty_like(send_elems)
    dist.all_to_all_single(recv_elems, send_elems, group=group)
    displs = torch.cumsum(recv_elems, 0) - recv_elems
    meta[2].copy_(_to_u32_bits(recv_elems))
    meta[3].copy_(_to_u32_bits(displs))
    return Route(send_rows=send_rows, recv_rows=[int(v) // hidden for v in recv_elems.tolist()],
                 send_offsets=send_offsets,
                 recv_offsets=[int(v) // hidden for v in displs.tolist()])


def put_offsets(route: Route, group=None) -> list[int]:
    """First row of this rank's block in every rank's receive buffer, for
    moe_permute_to_peers: rank d tells each source s where s's rows start in
    d's buffer (its receive displacement of s, meta row 3 / H), through one
    all-to-all."""
    S = _world(group)
    if len(route.recv_offsets) != S:
        raise ValueError("route does not match the group")
    mine = torch.tensor(route.recv_offsets, dtype=torch.int64)
    got = torch.empty_like(mine)
    dist.all_to_all_single(got, mine, group=group)
    return [int(v) for v in got.tolist()]


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


def _grouped_exchange(send: torch.Tensor, send_rows, send_offsets, recv: torch.Tensor,
                      recv_rows, recv_offsets, group=None) -> None:
    """Rows [send_offsets[p], +send_rows[p]) of `send` go to rank p, rows
    [recv_offsets[p], +recv_rows[p]) of `recv` come from rank p: one grouped
    batch of point-to-point transfers, this rank's own segment copied."""
    me = dist.get_rank(group)
    ops = []
    for peer in range(_world(group)):
        so, sn = send_offsets[peer], send_rows[peer]
        ro, rn = recv_offsets[peer], recv_rows[peer]
        if peer == me:
            if sn != rn:
                raise RuntimeError("own segment: send and receive counts differ")
            recv[ro:ro + rn].copy_(send[so:so + sn])
            continue
        dst = peer if group is None else dist.get_global_rank(group, peer)
        if sn > 0:
            ops.append(dist.P2POp(dist.isend, send[so:so + sn], dst, group))
        if rn > 0:
            ops.append(dist.P2POp(dist.irecv, recv[ro:ro + rn], dst, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def dispatch_exchange(rows: torch.Tensor, route: Route, group=None) -> torch.Tensor:
    """Ship segment s of `rows` (the dispatch output, or its code or scale
    rows) to rank s; returns the received rows, source rank by source rank."""
    if rows.shape[0] < max((o + n for o, n in zip(route.send_offsets, route.send_rows)),
                           default=0):
        raise ValueError("fewer rows than the route sends")
    send = _row_bytes(rows)
    out = torch.empty((route.recv_total, send.shape[1]), dtype=torch.uint8, device=rows.device)
    _grouped_exchange(send, route.send_rows, route.send_offsets, out, route.recv_rows,
                      route.recv_offsets, group)
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
    end = max((o + n for o, n in zip(route.send_offsets, route.send_rows)), default=0)
    if out is None:
        out = torch.zeros((end,) + tuple(expert_rows.shape[1:]),
                          dtype=expert_rows.dtype, device=expert_rows.device)
    if out.shape[0] < end or not out.is_contiguous():
        raise ValueError("out is not a contiguous buffer of the dispatch output's rows")
    if out.dtype != expert_rows.dtype or out.shape[1:] != expert_rows.shape[1:]:
        raise ValueError("out's rows differ from the expert rows in dtype or shape")
    # the reverse route: receive straight into the rows the segments left
    _grouped_exchange(_row_bytes(expert_rows), route.recv_rows, route.recv_offsets,
                      _row_bytes(out), route.send_rows, route.send_offsets, group)
    return out
