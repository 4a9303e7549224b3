"""Sharded prefill of one long sequence (block_sparse_streaming_b200.parallel),
host side on CPU: the shard plan covers the sequence, and with gloo ranks the
halo / sink exchange plus a prefill of each rank's local sequence reproduces
the whole-sequence result. The compute here is the fp64 oracle; the GPU test
emulates the ranks on one device with the CUDA prefill."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_streaming_b200 import parallel as par


@pytest.mark.parametrize("seq_len,world,n_sink", [(1957, 2, 1), (2765, 3, 1), (4096, 4, 1), (2900, 2, 2)])
def test_shard_plan_partitions_the_sequence(seq_len, world, n_sink):
    plans = [par.shard_plan(seq_len, world, r, n_sink, 7) for r in range(world)]
    rows = [p.own_rows for p in plans]
    assert rows[0][0] == 0 and rows[-1][1] == seq_len
    for (a0, a1), (b0, b1) in zip(rows, rows[1:]):
        assert a1 == b0 and a0 < a1
    for p in plans:
        # blocks of 128: the prefix is exactly s + l - 1 blocks, no gap
        assert p.pre_rows == (0 if p.rank == 0 else (n_sink + 6) * 128)
        assert p.local_len == p.pre_rows + (p.own_rows[1] - p.own_rows[0])


def test_shard_plan_rejects_small_shares():
    with pytest.raises(ValueError):
        par.shard_plan(6 * 128, 2, 0)          # 3 blocks per rank < s + l - 1
    with pytest.raises(ValueError):
        par.shard_plan(17 * 128, 3, 0)         # the last rank would get nothing
    with pytest.raises(ValueError):
        par.shard_plan(4096, 2, 0, 1, -1)      # unbounded window does not shard
    with pytest.raises(ValueError):
        par.shard_plan(4096, 2, 0, 1, 7, 96)   # block size not a power of two
    with pytest.raises(ValueError):
        par.shard_plan(700, 2, 0, 16, 300, 1)  # prefix 512 rows > 384-row shares


T = 128


def _lo(i, b, l):
    return max(0, (i // b - l + 1) * b)


def _visible(i, t, b, s, l):
    return t <= i and (t < s * b or t >= _lo(i, b, l))


def _walk(qb, b, s, l):
    """Key tiles a query tile walks, in order: the sink tiles, then the local ones."""
    sinks = min((s * b + T - 1) // T, qb + 1)
    first = max(sinks, _lo(qb * T, b, l) // T)
    return list(range(sinks)), list(range(first, qb + 1))


GENERAL = [(1, 16, 300), (64, 2, 14), (256, 1, 3), (32, 3, 20), (512, 1, 2), (2, 0, 100), (128, 1, 7), (16, 5, 1)]


@pytest.mark.parametrize("b,s,l", GENERAL)
def test_local_sequence_walks_the_same_tiles(b, s, l):
    """For every own query row of every rank, the local sequence's key tiles,
    walked in the kernels' order, are the whole sequence's tiles shifted by a
    whole number of tiles (sink tiles unshifted), and inside each tile the
    visible (query, key) pairs map one to one onto the whole sequence's, with
    no gap row visible: so each own row sums the same keys in the same order."""
    world = 3
    unit = max(b, T)
    seq_len = 3 * max(unit, 4 * T) * ((par.shard_plan(10 ** 6, 2, 1, s, l, b).pre_rows + unit - 1) // unit) - 77
    for r in range(1, world):
        p = par.shard_plan(seq_len, world, r, s, l, b)
        assert p.pre_rows % T == 0 and p.row0 % unit == 0 and p.pre_rows % b == 0
        shift = (p.row0 - p.pre_rows) // T
        gap0, halo0 = p.sink_rows, p.pre_rows - p.halo_rows

        def to_global(t):  # a local key row, as a whole-sequence row (None: a gap row)
            if t < gap0:
                return t
            if t < halo0:
                return None
            return t - p.pre_rows + p.row0

        for qb_loc in range(p.pre_rows // T, (p.local_len + T - 1) // T):
            qb = qb_loc + shift
            sk_loc, lo_loc = _walk(qb_loc, b, s, l)
            sk, lo = _walk(qb, b, s, l)
            assert sk_loc == sk and [kb + shift for kb in lo_loc] == lo
            for kb_loc, kb in zip(sk_loc + lo_loc, sk + lo):
                for i_loc in range(qb_loc * T, min(p.local_len, qb_loc * T + T)):
                    i = i_loc - p.pre_rows + p.row0
                    for off in range(T):
                        t_loc, t = kb_loc * T + off, kb * T + off
                        seen = _visible(i_loc, t_loc, b, s, l)
                        if seen:
                            assert to_global(t_loc) == t
                        assert seen == _visible(i, t, b, s, l)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case(seq_len, seed, H=2, d=64):
    import synth
    g = synth.rng(seed)
    return (synth.normal_bits(g, (seq_len, H, d)), synth.normal_bits(g, (seq_len, H, d)),
            synth.normal_bits(g, (seq_len, H, d)))


def _worker(rank, world, port, seq_len, n_sink, out_dir, block=128, n_local=7):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _case(seq_len, 77)
        plan = par.shard_plan(seq_len, world, rank, n_sink, n_local, block)
        lo, hi = plan.own_rows
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a[lo:hi]).view(np.int16))  # bf16 bits
        k_loc = par.exchange_kv(as_t(k), plan).numpy().view(np.uint16)
        v_loc = par.exchange_kv(as_t(v), plan).numpy().view(np.uint16)
        q_loc = par.local_queries(as_t(q), plan).numpy().view(np.uint16)
        cu = np.array([0, plan.local_len], np.int32)
        o, lse = oracle.forward(q_loc, k_loc, v_loc, cu, 2, 2, block, n_sink, n_local, 0.125)
        off = plan.pre_rows
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o[off:])
        np.save(os.path.join(out_dir, f"l{rank}.npy"), lse[off:])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("seq_len,world,n_sink,block,n_local", [
    (1957, 2, 1, 128, 7), (2765, 3, 1, 128, 7), (2900, 2, 2, 128, 7),
    (1500, 2, 16, 1, 300), (2300, 2, 2, 64, 14), (2000, 2, 1, 256, 3)])
def test_sharded_prefill_equals_whole_sequence(tmp_path, oracle_mod, seq_len, world, n_sink, block, n_local):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seq_len, n_sink, str(tmp_path), block, n_local))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    o = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)])
    lse = np.concatenate([np.load(tmp_path / f"l{r}.npy") for r in range(world)])
    q, k, v = _case(seq_len, 77)
    o_ref, lse_ref = oracle_mod.forward(q, k, v, np.array([0, seq_len], np.int32), 2, 2, block, n_sink, n_local,
                                        0.125)
    # the same keys in the same order for every query: identical fp64 results
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def _bwd_case(seq_len):
    import synth
    g = synth.rng(78)
    return tuple(synth.normal_bits(g, (seq_len, 1, 32)) for _ in range(4))  # q, k, v, dO


def _bwd_worker(rank, world, port, seq_len, n_sink, n_local, out_dir, block=128):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, do = _bwd_case(seq_len)
        plan = par.shard_plan(seq_len, world, rank, n_sink, n_local, block)
        lo, hi = plan.own_rows
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a[lo:hi]).view(np.int16))
        bits = lambda t: t.numpy().view(np.uint16)
        k_loc = bits(par.exchange_kv(as_t(k), plan))
        v_loc = bits(par.exchange_kv(as_t(v), plan))
        q_loc = bits(par.local_rows(as_t(q), plan))
        do_loc = bits(par.local_rows(as_t(do), plan))
        cu = np.array([0, plan.local_len], np.int32)
        dq, dk, dv = oracle.backward(q_loc, k_loc, v_loc, do_loc, cu, 1, 1, block, n_sink, n_local, 0.2)
        dk_own, dv_own = par.settle_key_grads(torch.from_numpy(dk), torch.from_numpy(dv), plan)
        off = plan.pre_rows
        np.save(os.path.join(out_dir, f"dq{rank}.npy"), dq[off:])
        np.save(os.path.join(out_dir, f"dk{rank}.npy"), dk_own.numpy())
        np.save(os.path.join(out_dir, f"dv{rank}.npy"), dv_own.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("seq_len,world,n_sink,n_local,block", [(1100, 2, 2, 3, 128), (1700, 3, 1, 3, 128),
                                                                (700, 2, 3, 5, 32), (1300, 2, 1, 2, 256)])
def test_sharded_backward_equals_whole_sequence(tmp_path, oracle_mod, seq_len, world, n_sink, n_local, block):
    """dQ of the own rows is exact; dK, dV of the own rows plus the halo
    gradients returned by the right neighbour and the sink gradients reduced
    onto rank 0 equal the whole sequence's (sums in fp32 here). A narrow
    window keeps the fp64 oracle backward short."""
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, seq_len, n_sink, n_local, str(tmp_path), block))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    cat = lambda name: np.concatenate([np.load(tmp_path / f"{name}{r}.npy") for r in range(world)])
    q, k, v, do = _bwd_case(seq_len)
    dq_ref, dk_ref, dv_ref = oracle_mod.backward(q, k, v, do, np.array([0, seq_len], np.int32), 1, 1, block, n_sink,
                                                 n_local, 0.2)
    assert np.array_equal(cat("dq"), dq_ref)
    for got, ref in ((cat("dk"), dk_ref), (cat("dv"), dv_ref)):
        assert np.abs(got - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
