"""Parity at the workloads' full sizes, on sampled outputs.

Inputs are drawn on the device by the seeded generators (synth) exactly as
bench.py draws them, the CUDA path runs through the C ABI in the same launch
configuration bench.py times, and the fp64 oracle evaluates the sampled rows
from a host copy of the same bits.
"""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, from_dev

pytestmark = pytest.mark.gpu


def bits(t):
    """bf16 device tensor -> numpy uint16 bit patterns on the host."""
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def sampled_rows(L, n, seed):
    rs = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 1023, 1024, 1025, L // 2, L - 129, L - 128, L - 1]
    return np.unique(np.concatenate([fixed, rs.choice(L, n, replace=False)])).astype(np.int64)


@pytest.mark.parametrize("L", [32768, 262144])
def test_absorbed_prefill_full_length(bss, oracle_mod, L):
    """Workload 2 (L = 32,768) and workload 4's prefill (L = 262,144): 64 heads,
    latent 576 with V = its first 512 columns, scale 1/sqrt(192)."""
    import torch
    H, D, DV = 64, 576, 512
    dev = torch.device("cuda")
    seed = synth.workload_seed(2 if L == 32768 else 4) * 1000
    q = synth.torch_normal_bf16((L, H, D), seed, dev)
    lat = synth.torch_normal_bf16((L, 1, D), seed + 1, dev)
    cu = torch.tensor([0, L], dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(192.0)
    out, lse = bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], cu, L, bss.Params(scale))
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    rows = sampled_rows(L, 48, L)
    q_host = np.empty((L, H, D), np.uint16)           # only the sampled rows are read (and touched)
    q_host[rows] = bits(q[torch.from_numpy(rows).to(dev)])
    lat_host = bits(lat)
    o_ref, lse_ref = oracle_mod.forward(q_host, lat_host, np.ascontiguousarray(lat_host[:, :, :DV]),
                                        synth.cu_seqlens([L]), H, 1, 128, 1, 7, scale, rows=rows)
    idx = torch.from_numpy(rows).to(dev)
    assert_close_o(from_dev(out[idx]), o_ref, f"prefill L={L}")
    assert_close_lse(lse[idx].cpu().numpy().astype(np.float64), lse_ref, f"prefill L={L}")


def test_training_workload_lengths(bss, oracle_mod):
    """Workload 5's drawn lengths (8 sequences, 684,193 tokens), 192/128 head
    dims, scale 1/sqrt(192); 8 heads here (heads are independent grid rows),
    forward and backward on sampled rows, including the sink rows of the two
    shortest sequences, which every later query block reads."""
    import torch
    w = synth.WORKLOADS[5]
    g = synth.rng(synth.workload_seed(5))
    lens = synth.loguniform_lengths(g, w["batch"], w["len_lo"], w["len_hi"], w["total_cap"])
    T, H, DQK, DV = int(lens.sum()), 8, 192, 128
    dev = torch.device("cuda")
    base = synth.workload_seed(5) * 1000 + 7
    q = synth.torch_normal_bf16((T, H, DQK), base + 1, dev)
    k = synth.torch_normal_bf16((T, H, DQK), base + 2, dev)
    v = synth.torch_normal_bf16((T, H, DV), base + 3, dev)
    do = synth.torch_normal_bf16((T, H, DV), base + 4, dev)
    cu_h = synth.cu_seqlens(lens)
    cu = torch.from_numpy(cu_h).to(dev)
    scale = w["scale"]
    p = bss.Params(scale)
    out, lse = bss.loza_ssa_prefill(q, k, v, cu, int(lens.max()), p)
    dq, dk, dv = bss.loza_ssa_backward(q, k, v, out, do, lse, cu, int(lens.max()), p)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    qh, kh, vh, doh = bits(q), bits(k), bits(v), bits(do)
    rs = np.random.default_rng(55)
    q_rows = np.unique(np.concatenate([cu_h[:-1], cu_h[1:] - 1, rs.choice(T, 40, replace=False)])).astype(np.int64)
    o_ref, lse_ref = oracle_mod.forward(qh, kh, vh, cu_h, H, H, 128, 1, 7, scale, rows=q_rows)
    qi = torch.from_numpy(q_rows).to(dev)
    assert_close_o(from_dev(out[qi]), o_ref, "training forward")
    assert_close_lse(lse[qi].cpu().numpy().astype(np.float64), lse_ref, "training forward LSE")
    short = np.argsort(lens)[:2]
    sink_rows = [int(cu_h[n]) + r for n in short for r in (0, 63, 127)]
    other = [int(cu_h[n]) + int(lens[n]) // 2 for n in range(len(lens))] + [int(cu_h[n]) + 128 for n in range(len(lens))]
    k_rows = np.unique(np.array(sink_rows + other, np.int64))
    rq, rk, rv = oracle_mod.backward(qh, kh, vh, doh, cu_h, H, H, 128, 1, 7, scale, q_rows=q_rows, k_rows=k_rows)
    ki = torch.from_numpy(k_rows).to(dev)
    for name, got, ref in (("dQ", dq[qi], rq), ("dK", dk[ki], rk), ("dV", dv[ki], rv)):
        got = from_dev(got)
        err = np.abs(got - ref)
        assert np.isfinite(got).all(), name
        assert err.max() <= 1e-2 * max(1.0, float(np.abs(ref).max())), f"{name}: max-abs {err.max():.3e}"
        assert err.mean() <= 1e-3 * max(1.0, float(np.abs(ref).mean())), f"{name}: mean-abs {err.mean():.3e}"


def test_absorbed_prefill_bitwise_repeatable(bss):
    """Workload 4's prefill length run three times: every output bit equal.
    The kernel keeps no atomics in its arithmetic, so any difference between
    runs exposes a synchronisation race between its pipeline roles."""
    import torch
    L, H, D, DV = 262144, 64, 576, 512
    dev = torch.device("cuda")
    seed = synth.workload_seed(4) * 1000 + 3
    q = synth.torch_normal_bf16((L, H, D), seed, dev)
    lat = synth.torch_normal_bf16((L, 1, D), seed + 1, dev)
    cu = torch.tensor([0, L], dtype=torch.int32, device=dev)
    p = bss.Params(1.0 / math.sqrt(192.0))
    o0, l0 = bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], cu, L, p)
    for _ in range(2):
        o1, l1 = bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], cu, L, p)
        torch.cuda.synchronize()
        assert bss.device_status() == 0
        bad_o = int((o1.view(torch.int16) != o0.view(torch.int16)).sum())
        bad_l = int((l1.view(torch.int32) != l0.view(torch.int32)).sum())
        assert bad_o == 0 and bad_l == 0, f"runs differ: {bad_o} O elements, {bad_l} LSE entries"
        del o1, l1
