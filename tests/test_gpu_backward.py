"""GPU parity of the SSA backward (dQ, dK, dV) against the fp64 oracle.

Tolerance per tensor (the pages fix none for gradients; see the design notes):
max-abs <= 1e-2 * max(1, max|ref|) and mean-abs <= 1e-3 * max(1, mean|ref|).
The forward O and LSE fed to the backward come from the GPU forward, as in
training; the oracle recomputes everything in fp64 from the inputs.
"""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_grad, from_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def run_bwd(bss, seed, lens, H, dqk, dv, scale, n_sink=1, n_local=7, block=128):
    import torch
    g = synth.rng(seed)
    T = int(sum(lens))
    cu = synth.cu_seqlens(lens)
    q = synth.normal_bits(g, (T, H, dqk))
    k = synth.normal_bits(g, (T, H, dqk))
    v = synth.normal_bits(g, (T, H, dv))
    do = synth.normal_bits(g, (T, H, dv))
    params = bss.Params(scale, block, n_sink, n_local)
    cu_d = torch.from_numpy(cu).cuda()
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    out, lse = bss.loza_ssa_prefill(qd, kd, vd, cu_d, max(lens), params)
    dq, dk, dvv = bss.loza_ssa_backward(qd, kd, vd, out, dod, lse, cu_d, max(lens), params)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    return (q, k, v, do, cu), (from_dev(dq), from_dev(dk), from_dev(dvv))


@pytest.mark.parametrize("dqk,dv,lens", [
    (64, 64, [1000, 300, 129]),
    (64, 64, [1]),
    (192, 128, [2100, 700, 1]),
])
def test_backward_full_oracle(bss, oracle_mod, dqk, dv, lens):
    H = 2
    scale = 1 / 8 if dqk == 64 else 1 / math.sqrt(192)
    (q, k, v, do, cu), (dq, dk, dvv) = run_bwd(bss, 101 + dqk, lens, H, dqk, dv, scale)
    rq, rk, rv = oracle_mod.backward(q, k, v, do, cu, H, H, 128, 1, 7, scale)
    assert_close_grad(dq, rq, "dQ")
    assert_close_grad(dk, rk, "dK")
    assert_close_grad(dvv, rv, "dV")


@pytest.mark.parametrize("n_sink,n_local", [(2, 3), (0, 2)])
def test_backward_other_windows(bss, oracle_mod, n_sink, n_local):
    lens = [1500, 260]
    (q, k, v, do, cu), (dq, dk, dvv) = run_bwd(bss, 107, lens, 2, 64, 64, 0.125, n_sink, n_local)
    rq, rk, rv = oracle_mod.backward(q, k, v, do, cu, 2, 2, 128, n_sink, n_local, 0.125)
    assert_close_grad(dq, rq, "dQ")
    assert_close_grad(dk, rk, "dK")
    assert_close_grad(dvv, rv, "dV")


def test_backward_long_sequence_sampled(bss, oracle_mod):
    """40,000 tokens (313 query blocks): the sink block's far part spans two
    partial chunks. dQ on 64 sampled rows; dK/dV on the sink rows and on rows of
    ordinary blocks."""
    L, H, dqk, dv = 40000, 1, 192, 128
    scale = 1 / math.sqrt(192)
    (q, k, v, do, cu), (dq, dk, dvv) = run_bwd(bss, 109, [L], H, dqk, dv, scale)
    rs = np.random.default_rng(5)
    qr = np.sort(rs.choice(L, 64, replace=False))
    kr = np.array([0, 77, 127, 128, 5000, 20000, 39999] + list(rs.choice(L, 5, replace=False)))
    rq, rk, rv = oracle_mod.backward(q, k, v, do, cu, H, H, 128, 1, 7, scale, q_rows=qr, k_rows=kr)
    assert_close_grad(dq[qr], rq, "dQ rows")
    assert_close_grad(dk[kr], rk, "dK rows")
    assert_close_grad(dvv[kr], rv, "dV rows")


def test_backward_is_deterministic(bss):
    lens = [3000, 500]
    _, a = run_bwd(bss, 111, lens, 2, 192, 128, 0.07)
    _, b = run_bwd(bss, 111, lens, 2, 192, 128, 0.07)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# general windows (any power-of-two block size; b = 1 is page 4's token window)
WINDOWS = [(1, 16, 1024), (64, 2, 14), (32, 3, 20), (256, 1, 3), (1, 0, 300), (16, 5, 30)]


@pytest.mark.parametrize("win", WINDOWS, ids=[f"b{w[0]}-s{w[1]}-l{w[2]}" for w in WINDOWS])
@pytest.mark.parametrize("dqk,dv,lens", [(64, 64, [3000, 700, 1, 129]), (192, 128, [2100, 300])])
def test_backward_general_windows(bss, oracle_mod, win, dqk, dv, lens):
    """Every row for windows of up to 512 keys; for the wider ones (the
    oracle's cost grows with the window squared) 300 sampled query rows and
    300 key rows, among them the sink keys and their neighbours, tile edges
    and each sequence's first and last rows."""
    b, s, l = win
    H = 2
    scale = 1 / 8 if dqk == 64 else 1 / math.sqrt(192)
    (q, k, v, do, cu), (dq, dk, dvv) = run_bwd(bss, 120 + b + dqk, lens, H, dqk, dv, scale, s, l, b)
    T = int(sum(lens))
    if (s + l) * b <= 512:
        qr = kr = np.arange(T)
    else:
        rs = np.random.default_rng(b + dqk)
        starts = synth.cu_seqlens(lens)[:-1]
        edges = [st + o for st, L in zip(starts, lens) for o in (0, 1, 15, 16, 17, 127, 128, L - 1) if o < L]
        qr = np.unique(np.concatenate([edges, rs.choice(T, 300, replace=False)]))
        kr = np.unique(np.concatenate([edges, rs.choice(T, 300, replace=False)]))
    rq, rk, rv = oracle_mod.backward(q, k, v, do, cu, H, H, b, s, l, scale, q_rows=qr, k_rows=kr)
    assert_close_grad(dq[qr], rq, f"dQ {win}")
    assert_close_grad(dk[kr], rk, f"dK {win}")
    assert_close_grad(dvv[kr], rv, f"dV {win}")


@pytest.mark.parametrize("win", [(1, 16, 1024), (64, 2, 14)], ids=["tokens-16-1024", "b64-2-14"])
def test_backward_general_windows_long_sampled(bss, oracle_mod, win):
    """40,000 tokens: the sink tile's far query tiles span two partial chunks;
    dQ on sampled rows, dK/dV on the sink keys, the keys just past them and
    rows of ordinary tiles."""
    b, s, l = win
    L, H, dqk, dv = 40000, 1, 192, 128
    scale = 1 / math.sqrt(192)
    (q, k, v, do, cu), (dq, dk, dvv) = run_bwd(bss, 130 + b, [L], H, dqk, dv, scale, s, l, b)
    rs = np.random.default_rng(6)
    qr = np.sort(rs.choice(L, 64, replace=False))
    kr = np.array([0, 15, 16, 17, 127, 128, 129, 5000, 20000, 39999] + list(rs.choice(L, 5, replace=False)))
    rq, rk, rv = oracle_mod.backward(q, k, v, do, cu, H, H, b, s, l, scale, q_rows=qr, k_rows=kr)
    assert_close_grad(dq[qr], rq, f"dQ rows {win}")
    assert_close_grad(dk[kr], rk, f"dK rows {win}")
    assert_close_grad(dvv[kr], rv, f"dV rows {win}")


def test_backward_general_window_deterministic(bss):
    lens = [3000, 500]
    _, a = run_bwd(bss, 140, lens, 2, 192, 128, 0.07, 16, 1024, 1)
    _, c = run_bwd(bss, 140, lens, 2, 192, 128, 0.07, 16, 1024, 1)
    for x, y in zip(a, c):
        np.testing.assert_array_equal(x, y)
