"""Sharding one long sequence's SSA prefill over ranks (one process per GPU).

Rank r owns the query blocks [j0, j1) of the sequence (contiguous, equal
shares of whole 128-token blocks) and the K/V rows of those blocks. A query in
block j reads the sink blocks 0 .. s-1 and the local blocks j-l+1 .. j (page 1
section 01 of the LoZA pages), so the rank also needs

    the sink blocks 0 .. s-1          (broadcast from rank 0) and
    the halo blocks j0-l+1 .. j0-1    (sent by the left neighbour),

one exchange before any compute. It then runs the one-GPU prefill on a local
sequence [sinks | halo | own blocks]: local block t = j - j0 + s + l - 1 of an
own block j has the window {0 .. s-1} U {t-l+1 .. t}, which is exactly the
sinks, the halo and the own blocks up to j, so the outputs of the own rows are
those of the whole-sequence prefill. The query rows of the prepended blocks are
zeros; their outputs are dropped (s + l - 1 blocks per rank).

The exchange uses torch.distributed point-to-point send/recv and broadcast
(NCCL over NVLink on GPUs, gloo on CPU) into each rank's own memory; kernels
only ever read local memory. Every rank's share must hold at least s + l - 1
blocks, so a halo never reaches past the left neighbour and a rank's halo
never overlaps the sinks.
"""
from __future__ import annotations

from dataclasses import dataclass

BLOCK = 128


@dataclass(frozen=True)
class ShardPlan:
    rank: int
    world: int
    j0: int          # first own query block
    j1: int          # one past the last own query block (clipped to the sequence)
    n_pre: int       # blocks prepended to the local sequence (0 on rank 0)
    seq_len: int

    @property
    def own_rows(self):
        return self.j0 * BLOCK, min(self.j1 * BLOCK, self.seq_len)

    @property
    def local_len(self):
        lo, hi = self.own_rows
        return self.n_pre * BLOCK + (hi - lo)


def shard_plan(seq_len: int, world: int, rank: int, n_sink: int = 1, n_local: int = 7) -> ShardPlan:
    """Equal shares of whole blocks (the last rank takes the ragged tail)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    if n_local < 1 or n_sink < 0:
        raise ValueError("sharding needs a bounded window (n_local >= 1)")
    nb = (seq_len + BLOCK - 1) // BLOCK
    per = (nb + world - 1) // world
    need = n_sink + n_local - 1
    if world > 1 and per < need:
        raise ValueError(f"each rank needs at least {need} blocks ({need * BLOCK} tokens)")
    if world > 1 and (world - 1) * per >= nb:
        raise ValueError("more ranks than shares of this sequence")
    j0 = min(rank * per, nb)
    j1 = min(j0 + per, nb)
    return ShardPlan(rank, world, j0, j1, 0 if j0 == 0 else need, seq_len)


def exchange_kv(kv_own, plan: ShardPlan, n_sink: int = 1, n_local: int = 7, group=None):
    """Assemble this rank's local K (or V, or latent) rows [sinks | halo | own]
    from its own rows (a [rows, ...] tensor of the own blocks, on this rank's
    device). Every rank must call it (collective: one broadcast, one
    send/recv pair per neighbour)."""
    import torch
    import torch.distributed as dist
    halo_rows = (n_local - 1) * BLOCK
    sink_rows = n_sink * BLOCK
    # rows travel as raw bytes, which every backend moves
    dtype = kv_own.dtype
    kv_own = kv_own.contiguous().view(torch.uint8)
    tail = kv_own.shape[1:]
    # sink blocks from rank 0 (its own first rows)
    sinks = torch.empty((sink_rows,) + tail, dtype=kv_own.dtype, device=kv_own.device)
    if plan.rank == 0:
        sinks.copy_(kv_own[:sink_rows])
    if plan.world > 1:
        dist.broadcast(sinks, src=0, group=group)
    # halo: the left neighbour's last l-1 blocks (its share is whole blocks, at least that many)
    halo = torch.empty((halo_rows,) + tail, dtype=kv_own.dtype, device=kv_own.device)
    ops = []
    if plan.world > 1:
        if plan.rank + 1 < plan.world:
            ops.append(dist.P2POp(dist.isend, kv_own[kv_own.shape[0] - halo_rows:].contiguous(), plan.rank + 1,
                                  group=group))
        if plan.rank > 0:
            ops.append(dist.P2POp(dist.irecv, halo, plan.rank - 1, group=group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
    if plan.n_pre == 0:
        return kv_own.view(dtype)
    return torch.cat([sinks, halo, kv_own], dim=0).view(dtype)


def local_kv_from_full(kv_full, plan: ShardPlan, n_sink: int = 1, n_local: int = 7):
    """The local rows [sinks | halo | own] that exchange_kv assembles, taken
    directly from the whole sequence's rows (for one process standing in for
    every rank)."""
    import torch
    lo, hi = plan.own_rows
    if plan.n_pre == 0:
        return kv_full[lo:hi]
    halo_lo = lo - (n_local - 1) * BLOCK
    return torch.cat([kv_full[: n_sink * BLOCK], kv_full[halo_lo:lo], kv_full[lo:hi]], dim=0)


def local_queries(q_own, plan: ShardPlan):
    """Local query rows: zeros for the prepended blocks, then the own rows."""
    import torch
    if plan.n_pre == 0:
        return q_own
    pre = torch.zeros((plan.n_pre * BLOCK,) + tuple(q_own.shape[1:]), dtype=q_own.dtype, device=q_own.device)
    return torch.cat([pre, q_own], dim=0)


def _require_block128(params):
    """The shard plan moves whole blocks of 128 tokens (the pages' b)."""
    if params.block_size != BLOCK:
        raise ValueError(f"sharding needs block_size {BLOCK}, got {params.block_size}")


def own_outputs(out_local, lse_local, plan: ShardPlan):
    """The rows of the own blocks in the local outputs."""
    off = plan.n_pre * BLOCK
    return out_local[off:], lse_local[off:]


def prefill_sharded(q_own, k_own, v_own, params, plan: ShardPlan, group=None, latent_v: bool = False):
    """SSA prefill of this rank's share of one sequence. q_own [rows, H, d_qk],
    k_own [rows, Hkv, d_qk], v_own [rows, Hkv, d_v] (or, with latent_v, the
    first d_v columns of k_own, which is then the absorbed latent cache).
    Returns (out, lse) of the own rows."""
    import torch
    from . import loza_ssa_prefill
    _require_block128(params)
    k_loc = exchange_kv(k_own, plan, params.n_sink, params.n_local, group)
    if latent_v:
        v_loc = k_loc[..., : v_own.shape[-1]]
    else:
        v_loc = exchange_kv(v_own, plan, params.n_sink, params.n_local, group)
    q_loc = local_queries(q_own, plan)
    cu = torch.tensor([0, q_loc.shape[0]], dtype=torch.int32, device=q_own.device)
    out, lse = loza_ssa_prefill(q_loc, k_loc, v_loc, cu, q_loc.shape[0], params)
    return own_outputs(out, lse, plan)


# ---------------------------------------------------------------------------
# Backward of the sharded prefill.
#
# Each rank runs the one-GPU backward on its local sequence [sinks | halo |
# own]: the prepended rows get zero dO (and zero O), so their queries add
# nothing to any gradient, and the own rows' dQ is exact. The key gradients of
# the prepended rows are partial sums that belong to other ranks:
#   halo rows (local blocks s .. s+l-2): the left neighbour's last l-1 blocks,
#       sent back to it and added to its own dK, dV;
#   sink rows (local blocks 0 .. s-1): every rank's share of the sink blocks'
#       gradients, summed onto rank 0 (which owns the sinks) by a reduce.
# The additions are done in fp32.
# ---------------------------------------------------------------------------
def local_rows(x_own, plan: ShardPlan):
    """Zero rows for the prepended blocks, then the own rows (q, out, dout, lse)."""
    return local_queries(x_own, plan)


def split_key_grads(dk_loc, dv_loc, plan: ShardPlan, n_sink: int = 1, n_local: int = 7):
    """The local backward's dK, dV (rows [sinks | halo | own]) as fp32 parts:
    (own dK, own dV, halo dK, halo dV, sink dK, sink dV); the halo and sink
    parts are None on rank 0, which has no prepended rows."""
    off = plan.n_pre * BLOCK
    own = (dk_loc[off:].float(), dv_loc[off:].float())
    if plan.n_pre == 0:
        return own + (None, None, None, None)
    s_rows, h_rows = n_sink * BLOCK, (n_local - 1) * BLOCK
    halo = (dk_loc[s_rows:s_rows + h_rows].float(), dv_loc[s_rows:s_rows + h_rows].float())
    sink = (dk_loc[:s_rows].float(), dv_loc[:s_rows].float())
    return own + halo + sink


def settle_key_grads(dk_loc, dv_loc, plan: ShardPlan, n_sink: int = 1, n_local: int = 7, group=None):
    """From the local backward's dK, dV (rows [sinks | halo | own]) return this
    rank's own dK, dV with the other ranks' contributions added (fp32 sums,
    then the input dtype): its right neighbour's halo part is added to its
    last l-1 blocks, and on rank 0 every rank's sink part to its first s
    blocks. Every rank must call it (collective)."""
    import torch
    import torch.distributed as dist
    out_dtype = dk_loc.dtype
    dk, dv, hk, hv, sk_part, sv_part = split_key_grads(dk_loc, dv_loc, plan, n_sink, n_local)
    halo_rows = (n_local - 1) * BLOCK
    sink_rows = n_sink * BLOCK
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
    _require_block128(params)
    k_loc = exchange_kv(k_own, plan, params.n_sink, params.n_local, group).contiguous()
    v_loc = exchange_kv(v_own, plan, params.n_sink, params.n_local, group).contiguous()
    q_loc = local_rows(q_own, plan).contiguous()
    o_loc = local_rows(out_own, plan).contiguous()
    do_loc = local_rows(dout_own, plan).contiguous()
    lse_loc = local_rows(lse_own, plan).contiguous()
    cu = torch.tensor([0, q_loc.shape[0]], dtype=torch.int32, device=q_own.device)
    dq, dk, dv = loza_ssa_backward(q_loc, k_loc, v_loc, o_loc, do_loc, lse_loc, cu, q_loc.shape[0], params)
    dk_own, dv_own = settle_key_grads(dk, dv, plan, params.n_sink, params.n_local, group)
    return dq[plan.n_pre * BLOCK:], dk_own, dv_own
