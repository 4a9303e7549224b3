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
from helpers import assert_close_grad, assert_close_lse, assert_close_o, from_dev

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


def window_rows(cu, n, i, b=128, s=1, l=7):
    """Packed rows of the keys query i (relative to sequence n) may read: whole
    selected blocks, cut at the sequence end (a superset of A(i); what the
    oracle needs in memory to evaluate row i)."""
    base, L = int(cu[n]), int(cu[n + 1] - cu[n])
    j = i // b
    blocks = sorted(set(range(min(s, j + 1))) | set(range(max(0, j - l + 1), j + 1)))
    return np.concatenate([np.arange(base + kb * b, base + min((kb + 1) * b, L)) for kb in blocks])


def readers_of_key(cu, n, t, b=128, s=1, l=7):
    """Query rows (relative to sequence n) whose windows select key t's block."""
    L = int(cu[n + 1] - cu[n])
    kb = t // b
    hi = L if kb < s else min(L, (kb + l) * b)
    return np.arange(t, hi)


def lazy_host_copy(t, rows):
    """Host array of t's full shape (bf16 bits) whose pages are touched only
    for the given packed rows, which hold t's values; the rest stay unbacked."""
    import torch
    host = np.empty(tuple(t.shape), np.uint16)
    rows = np.unique(np.asarray(rows, np.int64))
    for s0 in range(0, len(rows), 1 << 15):
        r = rows[s0:s0 + (1 << 15)]
        host[r] = bits(t[torch.from_numpy(r).to(t.device)])
    return host


def test_training_workload_full_shape(bss, oracle_mod):
    """Workload 5 as bench.py runs it: the eight drawn lengths (684,193 tokens
    packed by cu_seqlens), 64 heads, 192/128 head dims, scale 1/sqrt(192);
    q has 8.4 G elements, so every 64-bit index path of the forward and the
    backward is exercised. Forward and dQ on sampled query rows (each
    sequence's first and last row and random ones); dK and dV on the sink rows
    0 and 127 of the two shortest sequences (every query of the sequence
    reaches them) and on rows of ordinary blocks of every sequence."""
    import torch
    w = synth.WORKLOADS[5]
    g = synth.rng(synth.workload_seed(5))
    lens = synth.loguniform_lengths(g, w["batch"], w["len_lo"], w["len_hi"], w["total_cap"])
    T, H, DQK, DV = int(lens.sum()), w["n_heads"], w["d_qk"], w["d_v"]
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
    seq_of = lambda r: int(np.searchsorted(cu_h, r, side="right") - 1)
    rs = np.random.default_rng(55)
    q_rows = np.unique(np.concatenate([cu_h[:-1], cu_h[1:] - 1, rs.choice(T, 40, replace=False)])).astype(np.int64)
    short = np.argsort(lens)[:2]
    sink_rows = [int(cu_h[n]) + r for n in short for r in (0, 127)]
    other = [int(cu_h[n]) + int(lens[n]) // 2 for n in range(len(lens))] + [int(cu_h[n]) + 128 for n in short]
    k_rows = np.unique(np.array(sink_rows + other, np.int64))
    # rows the oracle reads: the sampled queries and their windows, and every
    # query reaching a sampled key with that query's window
    need_q = [q_rows]
    need_kv = [window_rows(cu_h, seq_of(r), r - int(cu_h[seq_of(r)])) for r in q_rows]
    for r in k_rows:
        n = seq_of(r)
        readers = readers_of_key(cu_h, n, int(r - cu_h[n]))
        need_q.append(readers + int(cu_h[n]))
        lo, hi = int(readers[0]), int(readers[-1])
        # the readers' windows: the sink block and the local blocks from lo's window start through hi
        need_kv.append(window_rows(cu_h, n, lo))
        need_kv.append(np.arange(int(cu_h[n]) + max(0, lo // 128 - 6) * 128, int(cu_h[n]) + hi + 1))
    need_q = np.unique(np.concatenate(need_q))
    need_kv = np.unique(np.concatenate(need_kv))
    qh, doh = lazy_host_copy(q, need_q), lazy_host_copy(do, need_q)
    kh, vh = lazy_host_copy(k, need_kv), lazy_host_copy(v, need_kv)
    o_ref, lse_ref = oracle_mod.forward(qh, kh, vh, cu_h, H, H, 128, 1, 7, scale, rows=q_rows)
    qi = torch.from_numpy(q_rows).to(dev)
    assert_close_o(from_dev(out[qi]), o_ref, "workload 5 forward, 64 heads")
    assert_close_lse(lse[qi].cpu().numpy().astype(np.float64), lse_ref, "workload 5 forward LSE, 64 heads")
    rq, rk, rv = oracle_mod.backward(qh, kh, vh, doh, cu_h, H, H, 128, 1, 7, scale, q_rows=q_rows, k_rows=k_rows)
    ki = torch.from_numpy(k_rows).to(dev)
    assert_close_grad(from_dev(dq[qi]), rq, "workload 5 dQ, 64 heads")
    assert_close_grad(from_dev(dk[ki]), rk, "workload 5 dK (sink and block rows), 64 heads")
    assert_close_grad(from_dev(dv[ki]), rv, "workload 5 dV (sink and block rows), 64 heads")


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
