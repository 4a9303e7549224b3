"""The sharded prefill on one B200: each rank's local sequence [sinks | halo |
own blocks] (assembled directly, as exchange_kv would) through the CUDA prefill
gives exactly the rows of the whole-sequence prefill."""
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


@pytest.mark.parametrize("shape,world,n_sink", [("absorbed", 3, 1), ("192/128", 2, 1), ("192/128", 3, 2),
                                                ("absorbed", 2, 2)])
def test_sharded_prefill_equals_whole(bss, shape, world, n_sink):
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
    params = bss.Params(1 / math.sqrt(192), 128, n_sink, 7)
    cu = torch.tensor([0, seq_len], dtype=torch.int32, device="cuda")
    out_full, lse_full = bss.loza_ssa_prefill(q, k, v, cu, seq_len, params)
    for r in range(world):
        plan = par.shard_plan(seq_len, world, r, n_sink, 7)
        lo, hi = plan.own_rows
        k_loc = par.local_kv_from_full(k, plan, n_sink, 7).contiguous()
        v_loc = k_loc[:, :, :512] if shape == "absorbed" else par.local_kv_from_full(v, plan, n_sink, 7).contiguous()
        q_loc = par.local_queries(q[lo:hi], plan).contiguous()
        cu_loc = torch.tensor([0, q_loc.shape[0]], dtype=torch.int32, device="cuda")
        out, lse = bss.loza_ssa_prefill(q_loc, k_loc, v_loc, cu_loc, q_loc.shape[0], params)
        out_own, lse_own = par.own_outputs(out, lse, plan)
        torch.cuda.synchronize()
        assert torch.equal(out_own, out_full[lo:hi]), f"rank {r} O"
        assert torch.equal(lse_own, lse_full[lo:hi]), f"rank {r} LSE"
