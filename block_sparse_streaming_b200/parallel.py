"""Sharding one long sequence's SSA prefill over ranks (one process per GPU).

The window of query i (page 1 section 01 of the LoZA pages, blocks of b
tokens) is the sink rows [0, s*b) and the local rows [lo(i), i] with
lo(i) = max(0, (floor(i/b) - l + 1) * b). Rank r owns the rows [row0, row1)
of the sequence (equal shares of whole units of U = max(b, 128) rows, so a
share starts on a block and on a kernel tile) and the K/V rows of those rows.
Its own queries then read

    the sink rows [0, s*b)                     (broadcast from rank 0) and
    the halo rows [row0 - (l-1)*b, row0)       (sent by the left neighbour),

one exchange before any compute. It runs the one-GPU prefill on a local
sequence

    [sinks (s*b) | gap (zeros) | halo ((l-1)*b) | own rows],

with the prefix (sinks, gap, halo) of P rows, P the smallest multiple of U that
holds the sinks rounded up to whole 128-row tiles plus the halo. An own row i
sits at local row i' = i - row0 + P. Because row0 and P are both multiples of U,
floor(i'/b) - floor(i/b) = (P - row0)/b, so the local window of i' is the sinks
plus [lo(i) - row0 + P, i']: the halo and the own rows up to i, the same keys
as in the whole sequence. The gap rows lie past the sinks and before every own
row's window, so no own query sees them. Because row0 and P are multiples of
128, each own row and key keeps its place inside its 128-row tile, and the
halo never shares a tile with the sinks (on either side). The kernels
therefore walk the same key tiles in the same order, and the own rows'
outputs are bit-identical to the whole-sequence prefill. The query rows of
the prefix are zeros; their outputs are dropped.

The exchange uses torch.distributed point-to-point send/recv and broadcast
(NCCL over NVLink on GPUs, gloo on CPU) into each rank's own memory; kernels
only ever read local memory. Every rank's share must hold at least P rows, so a
halo never reaches past the left neighbour and never overlaps the sink tiles.
"""
from __future__ import annotations

from dataclasses import dataclass

TILE = 128  # rows of a query / key tile of the kernels


@dataclass(frozen=True)
class ShardPlan:
    rank: int
    world: int
    row0: int        # first own row
    row1: int        # one past the last own row
    pre_rows: int    # rows of the local prefix [sinks | gap | halo] (0 on rank 0)
    seq_len: int
    sink_rows: int   # s * b
    halo_rows: int   # (l - 1) * b

    @property
    def own_rows(self):
        return self.row0, self.row1

    @property
    def local_len(self):
        return self.pre_rows + (self.row1 - self.row0)


def _round_up(x, m):
    return (x + m - 1) // m * m


def shard_plan(seq_len: int, world: int, rank: int, n_sink: int = 1, n_local: int = 7,
               block: int = 128) -> ShardPlan:
    """Equal shares of whole units of max(b, 128) rows (the last rank takes the ragged tail)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    if n_local < 1 or n_sink < 0:
        raise ValueError("sharding needs a bounded window (n_local >= 1)")
    if block < 1 or block & (block - 1):
        raise ValueError("block size must be a power of two")
    unit = max(block, TILE)
    sink_rows, halo_rows = n_sink * block, (n_local - 1) * block
    pre = _round_up(_round_up(sink_rows, TILE) + halo_rows, unit)
    n_units = (seq_len + unit - 1) // unit
    per = (n_units + world - 1) // world
    if world > 1 and per * unit < pre:
        raise ValueError(f"each rank needs at least {pre} rows")
    if world > 1 and (world - 1) * per >= n_units:
        raise ValueError("more ranks than shares of this sequence")
    row0 = min(rank * per * unit, seq_len)
    row1 = min(row0 + per * unit, seq_len)
    return ShardPlan(rank, world, row0, row1, 0 if row0 == 0 else pre, seq_len, sink_rows, halo_rows)


def _prefix(sinks, halo, plan: ShardPlan):
    """[sinks | gap of zero rows | halo], the local prefix."""
    import torch
    gap = plan.pre_rows - plan.sink_rows - plan.halo_rows
    zeros = torch.zeros((gap,) + tuple(sinks.shape[1:]), dtype=sinks.dtype, device=sinks.device)
    return torch.cat([sinks, zeros, halo], dim=0)


def exchange_kv(kv_own, plan: ShardPlan, group=None):
    """Assemble this rank's local K (or V, or latent) rows [sinks | gap | halo |
    own] from its own rows (a [rows, ...] tensor, on this rank's device).
    Every rank must call it (collective: one broadcast, one send/recv pair per
    neighbour)."""
    import torch
    import torch.distributed as dist
    # rows travel as raw bytes, which every backend moves
    dtype = kv_own.dtype
    kv_own = kv_own.contiguous().view(torch.uint8)
    tail = kv_own.shape[1:]
    # the sink rows from rank 0 (its own first rows)
    sinks = torch.empty((plan.sink_rows,) + tail, dtype=kv_own.dtype, device=kv_own.device)
    if plan.rank == 0:
        sinks.copy_(kv_own[:plan.sink_rows])
    if plan.world > 1:
        dist.broadcast(sinks, src=0, group=group)
    # the halo: the left neighbour's last (l-1)*b rows (its share holds at least that many)
    halo = torch.empty((plan.halo_rows,) + tail, dtype=kv_own.dtype, device=kv_own.device)
    ops = []
    if plan.world > 1:
        if plan.rank + 1 < plan.world:
            ops.append(dist.P2POp(dist.isend, kv_own[kv_own.shape[0] - plan.halo_rows:].contiguous(), plan.rank + 1,
                                  group=group))
        if plan.rank > 0:
            ops.append(dist.P2POp(dist.irecv, halo, plan.rank - 1, group=group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
    if plan.pre_rows == 0:
        return kv_own.view(dtype)
    return torch.cat([_prefix(sinks, halo, plan), kv_own], dim=0).view(dtype)


def local_kv_from_full(kv_full, plan: ShardPlan):
    """The local rows that exchange_kv assembles, taken directly from the
    whole sequence's rows (for one process standing in for every rank)."""
    import torch
    lo, hi = plan.own_rows
    if plan.pre_rows == 0:
        return kv_full[lo:hi]
    prefix = _prefix(kv_full[:plan.sink_rows], kv_full[lo - plan.halo_rows:lo], plan)
    return torch.cat([prefix, kv_full[lo:hi]], dim=0)


def local_queries(q_own, plan: ShardPlan):
    """Local query rows: zeros for the prefix, then the own rows."""
    import torch
    if plan.pre_rows == 0:
        return q_own
    pre = torch.zeros((plan.pre_rows,) + tuple(q_own.shape[1:]), dtype=q_own.dtype, device=q_own.device)
    return torch.cat([pre, q_own], dim=0)


def _check_params(params, plan: ShardPlan):
    """The plan must have been made for this window."""
    if (params.n_local < 1 or plan.sink_rows != params.n_sink * params.block_size or
            plan.halo_rows != (params.n_local - 1) * params.block_size):
        raise ValueError("shard plan made for another window")


def own_outputs(out_local, lse_local, plan: ShardPlan):
    """The own rows of the local outputs."""
    return out_local[plan.pre_rows:], lse_local[plan.pre_rows:]


def prefill_sharded(q_own, k_own, v_own, params, plan: ShardPlan, group=None, latent_v: bool = False):
    """SSA prefill of this rank's share of one sequence. q_own [rows, H, d_qk],
    k_own [rows, Hkv, d_qk], v_own [rows, Hkv, d_v] (or, with latent_v, the
    first d_v columns of k_own, which is then the absorbed latent cache).
    Returns (out, lse) of the own rows."""
    import torch
    from . import loza_ssa_prefill
    _check_params(params, plan)
    k_loc = exchange_kv(k_own, plan, group)
    if latent_v:
        v_loc = k_loc[..., : v_own.shape[-1]]
    else:
        v_loc = exchange_kv(v_own, plan, group)
    q_loc = local_queries(q_own, plan)
    cu = torch.tensor([0, q_loc.shape[0]], dtype=torch.int32, device=q_own.device)
    out, lse = loza_ssa_prefill(q_loc, k_loc, v_loc, cu, q_loc.shape[0], params)
    return own_outputs(out, lse, plan)


# ---------------------------------------------------------------------------
# Backward of the sharded prefill.
#
# Each rank runs the one-GPU backward on its local sequence [sinks | gap |
# halo | own]: the prefix rows get zero dO (and zero O), so their queries add
# nothing to any gradient, and the own rows' dQ is exact. The key gradients of
# the prefix rows are partial sums that belong to other ranks:
#   halo rows: the left neighbour's last (l-1)*b rows, sent back to it and
#       added to its own dK, dV;
#   sink rows: every rank's share of the sink rows' gradients, summed onto
#       rank 0 (which owns the sinks) by a reduce;
#   gap rows: seen by no query with a nonzero dO, so zero, and dropped.
# The additions are done in fp32.
# ---------------------------------------------------------------------------
def local_rows(x_own, plan: ShardPlan):
    """Zero rows for the prefix, then the own rows (q, out, dout, lse)."""
    return local_queries(x_own, plan)


def split_key_grads(dk_loc, dv_loc, plan: ShardPlan):
    """The local backward's dK, dV (rows [sinks | gap | halo | own]) as fp32
    parts: (own dK, own dV, halo dK, halo dV, sink dK, sink dV); the halo and
    sink parts are None on rank 0, which has no prefix."""
    off = plan.pre_rows
    own = (dk_loc[off:].float(), dv_loc[off:].float())
    if off == 0:
        return own + (None, None, None, None)
    h0 = off - plan.halo_rows
    halo = (dk_loc[h0:off].float(), dv_loc[h0:off].float())
    sink = (dk_loc[:plan.sink_rows].float(), dv_loc[:plan.sink_rows].float())
    return own + halo + sink


def settle_key_grads(dk_loc, dv_loc, plan: ShardPlan, group=None):
    """From the local backward's dK, dV (rows [sinks | gap | halo | own])
    return this rank's own dK, dV with the other ranks' contributions added
    (fp32 sums, then the input dtype): its right neighbour's halo part is added
    to its last (l-1)*b rows, and on rank 0 every rank's sink part to its
    first s*b rows. Every rank must call it (collective)."""
    import torch
    import torch.distributed as dist
    out_dtype = dk_loc.dtype
    dk, dv, hk, hv, sk_part, sv_part = split_key_grads(dk_loc, dv_loc, plan)
    halo_rows, sink_rows = plan.halo_rows, plan.sink_rows
    if plan.world > 1:
        ops = []
        recv_k = recv_v = None
        if plan.rank > 0:  # the halo gradients go back to the left neighbour
            ops.append(dist.P2POp(dist.isend, hk.contiguous(), plan.rank - 1, group=group))
            ops.append(dist.P2POp(dist.isend, hv.contiguous(), plan.rank - 1, group=group))
        if plan.rank + 1 < plan.world:
            recv_k = torch.empty((halo_rows,) + tuple(dk.shape[1:]), dtype=torch.float32, device=dk.device)
            recv_v = torch.empty((halo_rows,) + tuple(dv.shape[1:]), dtype=torch.float32, device=dv.device)
            ops.append(dist.P2POp(dist.irecv, recv_k, plan.rank + 1, group=group))
            ops.append(dist.P2POp(dist.irecv, recv_v, plan.rank + 1, group=group))
        for req in dist.batch_isend_irecv(ops):
            req.wait()
        if recv_k is not None:
            dk[dk.shape[0] - halo_rows:] += recv_k
            dv[dv.shape[0] - halo_rows:] += recv_v
        # the sink gradients of every other rank, summed onto rank 0
        sk = sk_part.contiguous() if sk_part is not None else torch.zeros(
            (sink_rows,) + tuple(dk.shape[1:]), dtype=torch.float32, device=dk.device)
        sv = sv_part.contiguous() if sv_part is not None else torch.zeros(
            (sink_rows,) + tuple(dv.shape[1:]), dtype=torch.float32, device=dv.device)
        dist.reduce(sk, dst=0, op=dist.ReduceOp.SUM, group=group)
        dist.reduce(sv, dst=0, op=dist.ReduceOp.SUM, group=group)
        if plan.rank == 0:
            dk[:sink_rows] += sk
            dv[:sink_rows] += sv
    return dk.to(out_dtype), dv.to(out_dtype)


def backward_sharded(q_own, k_own, v_own, out_own, dout_own, lse_own, params, plan: ShardPlan, group=None):
    """SSA backward of this rank's share of one sequence (per-head K, V).
    Returns (dq, dk, dv) of the own rows."""
    import torch
    from . import loza_ssa_backward
    _check_params(params, plan)
    k_loc = exchange_kv(k_own, plan, group).contiguous()
    v_loc = exchange_kv(v_own, plan, group).contiguous()
    q_loc = local_rows(q_own, plan).contiguous()
    o_loc = local_rows(out_own, plan).contiguous()
    do_loc = local_rows(dout_own, plan).contiguous()
    lse_loc = local_rows(lse_own, plan).contiguous()
    cu = torch.tensor([0, q_loc.shape[0]], dtype=torch.int32, device=q_own.device)
    dq, dk, dv = loza_ssa_backward(q_loc, k_loc, v_loc, o_loc, do_loc, lse_loc, cu, q_loc.shape[0], params)
    dk_own, dv_own = settle_key_grads(dk, dv, plan, group)
    return dq[plan.pre_rows:], dk_own, dv_own
