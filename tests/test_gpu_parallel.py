"""The sharded prefill on one B200: each rank's local sequence [sinks | gap |
halo | own rows] (assembled directly, as exchange_kv would) through the CUDA
prefill gives exactly the rows of the whole-sequence prefill, for blocks of 128
tokens and for general windows (other power-of-two block sizes)."""
import math

import numpy as np
import pytest

import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


@pytest.mark.parametrize("shape,world,n_sink,block,n_local", [
    ("absorbed", 3, 1, 128, 7), ("192/128", 2, 1, 128, 7), ("192/128", 3, 2, 128, 7), ("absorbed", 2, 2, 128, 7),
    ("absorbed", 3, 16, 1, 300), ("192/128", 2, 16, 1, 300), ("192/128", 3, 2, 64, 14), ("absorbed", 2, 1, 256, 3),
    ("192/128", 3, 3, 32, 20), ("absorbed", 2, 3, 32, 20)])
def test_sharded_prefill_equals_whole(bss, shape, world, n_sink, block, n_local):
    import torch
    from block_sparse_streaming_b200 import parallel as par
    seq_len, H = 5000, 4
    g = synth.rng(400 + world + n_sink)
    if shape == "absorbed":
        q = to_dev(synth.normal_bits(g, (seq_len, H, 576)))
        k = to_dev(synth.normal_bits(g, (seq_len, 1, 576)))
        v = k[:, :, :512]
    else:
        q = to_dev(synth.normal_bits(g, (seq_len, H, 192)))
        k = to_dev(synth.normal_bits(g, (seq_len, H, 192)))
        v = to_dev(synth.normal_bits(g, (seq_len, H, 128)))
    params = bss.Params(1 / math.sqrt(192), block, n_sink, n_local)
    cu = torch.tensor([0, seq_len], dtype=torch.int32, device="cuda")
    out_full, lse_full = bss.loza_ssa_prefill(q, k, v, cu, seq_len, params)
    for r in range(world):
        plan = par.shard_plan(seq_len, world, r, n_sink, n_local, block)
        lo, hi = plan.own_rows
        k_loc = par.local_kv_from_full(k, plan).contiguous()
        v_loc = k_loc[:, :, :512] if shape == "absorbed" else par.local_kv_from_full(v, plan).contiguous()
        q_loc = par.local_queries(q[lo:hi], plan).contiguous()
        cu_loc = torch.tensor([0, q_loc.shape[0]], dtype=torch.int32, device="cuda")
        out, lse = bss.loza_ssa_prefill(q_loc, k_loc, v_loc, cu_loc, q_loc.shape[0], params)
        out_own, lse_own = par.own_outputs(out, lse, plan)
        torch.cuda.synchronize()
        assert torch.equal(out_own, out_full[lo:hi]), f"rank {r} O"
        assert torch.equal(lse_own, lse_full[lo:hi]), f"rank {r} LSE"


@pytest.mark.parametrize("world,n_sink,block,n_local", [(2, 1, 128, 7), (3, 2, 128, 7), (2, 16, 1, 300),
                                                       (3, 2, 64, 14), (2, 1, 256, 3)])
def test_sharded_backward_matches_whole(bss, world, n_sink, block, n_local):
    """The sharded backward on one B200: every rank's local backward through
    the CUDA kernels, its key gradients split into own / halo / sink parts and
    summed as the collectives would. dQ is bit-identical to the whole
    sequence's; dK, dV (extra bf16 roundings of the summed parts) agree within
    the gradient tolerance."""
    import torch
    from block_sparse_streaming_b200 import parallel as par
    seq_len, H = 5000, 4
    g = synth.rng(500 + world)
    q, k = (to_dev(synth.normal_bits(g, (seq_len, H, 192))) for _ in range(2))
    v, dout = (to_dev(synth.normal_bits(g, (seq_len, H, 128))) for _ in range(2))
    params = bss.Params(1 / math.sqrt(192), block, n_sink, n_local)
    cu = torch.tensor([0, seq_len], dtype=torch.int32, device="cuda")
    out, lse = bss.loza_ssa_prefill(q, k, v, cu, seq_len, params)
    dq_ref, dk_ref, dv_ref = bss.loza_ssa_backward(q, k, v, out, dout, lse, cu, seq_len, params)
    plans = [par.shard_plan(seq_len, world, r, n_sink, n_local, block) for r in range(world)]
    parts = []
    for plan in plans:
        lo, hi = plan.own_rows
        loc = lambda x: par.local_rows(x[lo:hi], plan).contiguous()
        k_loc = par.local_kv_from_full(k, plan).contiguous()
        v_loc = par.local_kv_from_full(v, plan).contiguous()
        cu_loc = torch.tensor([0, plan.local_len], dtype=torch.int32, device="cuda")
        dq, dk, dv = bss.loza_ssa_backward(loc(q), k_loc, v_loc, loc(out), loc(dout), loc(lse), cu_loc, plan.local_len,
                                           params)
        assert torch.equal(dq[plan.pre_rows:], dq_ref[lo:hi]), f"rank {plan.rank} dQ"
        parts.append(par.split_key_grads(dk, dv, plan))
    # what the exchange does: halo parts to the left neighbour, sink parts onto rank 0
    dk_sum = [p[0].clone() for p in parts]
    dv_sum = [p[1].clone() for p in parts]
    h, sk = plans[0].halo_rows, plans[0].sink_rows
    for r in range(1, world):
        if h:
            dk_sum[r - 1][-h:] += parts[r][2]
            dv_sum[r - 1][-h:] += parts[r][3]
        dk_sum[0][:sk] += parts[r][4]
        dv_sum[0][:sk] += parts[r][5]
    dk_got = torch.cat([x.to(torch.bfloat16) for x in dk_sum]).double().cpu().numpy()
    dv_got = torch.cat([x.to(torch.bfloat16) for x in dv_sum]).double().cpu().numpy()
    for got, ref, name in ((dk_got, dk_ref.double().cpu().numpy(), "dK"), (dv_got, dv_ref.double().cpu().numpy(), "dV")):
        err = np.abs(got - ref)
        assert err.max() <= 1e-2 * max(1.0, np.abs(ref).max()), f"{name} max-abs {err.max()}"
        assert err.mean() <= 1e-3 * max(1.0, np.abs(ref).mean()), f"{name} mean-abs {err.mean()}"
