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
        assert p.n_pre == (0 if p.rank == 0 else n_sink + 6)
        assert p.local_len == p.n_pre * 128 + (p.own_rows[1] - p.own_rows[0])


def test_shard_plan_rejects_small_shares():
    with pytest.raises(ValueError):
        par.shard_plan(6 * 128, 2, 0)          # 3 blocks per rank < s + l - 1
    with pytest.raises(ValueError):
        par.shard_plan(17 * 128, 3, 0)         # the last rank would get nothing
    with pytest.raises(ValueError):
        par.shard_plan(4096, 2, 0, 1, -1)      # unbounded window does not shard


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


def _worker(rank, world, port, seq_len, n_sink, out_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _case(seq_len, 77)
        plan = par.shard_plan(seq_len, world, rank, n_sink, 7)
        lo, hi = plan.own_rows
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a[lo:hi]).view(np.int16))  # bf16 bits
        k_loc = par.exchange_kv(as_t(k), plan, n_sink, 7).numpy().view(np.uint16)
        v_loc = par.exchange_kv(as_t(v), plan, n_sink, 7).numpy().view(np.uint16)
        q_loc = par.local_queries(as_t(q), plan).numpy().view(np.uint16)
        cu = np.array([0, plan.local_len], np.int32)
        o, lse = oracle.forward(q_loc, k_loc, v_loc, cu, 2, 2, 128, n_sink, 7, 0.125)
        off = plan.n_pre * 128
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o[off:])
        np.save(os.path.join(out_dir, f"l{rank}.npy"), lse[off:])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("seq_len,world,n_sink", [(1957, 2, 1), (2765, 3, 1), (2900, 2, 2)])
def test_sharded_prefill_equals_whole_sequence(tmp_path, oracle_mod, seq_len, world, n_sink):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seq_len, n_sink, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    o = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)])
    lse = np.concatenate([np.load(tmp_path / f"l{r}.npy") for r in range(world)])
    q, k, v = _case(seq_len, 77)
    o_ref, lse_ref = oracle_mod.forward(q, k, v, np.array([0, seq_len], np.int32), 2, 2, 128, n_sink, 7, 0.125)
    # the same keys in the same order for every query: identical fp64 results
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def _bwd_case(seq_len):
    import synth
    g = synth.rng(78)
    return tuple(synth.normal_bits(g, (seq_len, 1, 32)) for _ in range(4))  # q, k, v, dO


def _bwd_worker(rank, world, port, seq_len, n_sink, n_local, out_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, do = _bwd_case(seq_len)
        plan = par.shard_plan(seq_len, world, rank, n_sink, n_local)
        lo, hi = plan.own_rows
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a[lo:hi]).view(np.int16))
        bits = lambda t: t.numpy().view(np.uint16)
        k_loc = bits(par.exchange_kv(as_t(k), plan, n_sink, n_local))
        v_loc = bits(par.exchange_kv(as_t(v), plan, n_sink, n_local))
        q_loc = bits(par.local_rows(as_t(q), plan))
        do_loc = bits(par.local_rows(as_t(do), plan))
        cu = np.array([0, plan.local_len], np.int32)
        dq, dk, dv = oracle.backward(q_loc, k_loc, v_loc, do_loc, cu, 1, 1, 128, n_sink, n_local, 0.2)
        dk_own, dv_own = par.settle_key_grads(torch.from_numpy(dk), torch.from_numpy(dv), plan, n_sink, n_local)
        off = plan.n_pre * 128
        np.save(os.path.join(out_dir, f"dq{rank}.npy"), dq[off:])
        np.save(os.path.join(out_dir, f"dk{rank}.npy"), dk_own.numpy())
        np.save(os.path.join(out_dir, f"dv{rank}.npy"), dv_own.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("seq_len,world,n_sink,n_local", [(1100, 2, 2, 3), (1700, 3, 1, 3)])
def test_sharded_backward_equals_whole_sequence(tmp_path, oracle_mod, seq_len, world, n_sink, n_local):
    """dQ of the own rows is exact; dK, dV of the own rows plus the halo
    gradients returned by the right neighbour and the sink gradients reduced
    onto rank 0 equal the whole sequence's (sums in fp32 here). A narrow
    window keeps the fp64 oracle backward short."""
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, seq_len, n_sink, n_local, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    cat = lambda name: np.concatenate([np.load(tmp_path / f"{name}{r}.npy") for r in range(world)])
    q, k, v, do = _bwd_case(seq_len)
    dq_ref, dk_ref, dv_ref = oracle_mod.backward(q, k, v, do, np.array([0, seq_len], np.int32), 1, 1, 128, n_sink,
                                                 n_local, 0.2)
    assert np.array_equal(cat("dq"), dq_ref)
    for got, ref in ((cat("dk"), dk_ref), (cat("dv"), dv_ref)):
        assert np.abs(got - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
