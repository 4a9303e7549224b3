"""GPU parity of the prefill and decode kernels under windows other than the
pages' (b, s, l) = (128, 1, 7), against the fp64 oracle on the same bits:

  * page 4's token-granular window (its streaming-aware index keeps 16 sink
    tokens and a 1,024-token sliding window): blocks of one token, b = 1,
    s = 16, l = 1024 (the oracle's block form with b = 1 is pinned to its
    token form in test_oracle_token_window.py);
  * other block sizes (b is the method's parameter, page 1 section 01 (1)):
    b = 64 with (s, l) = (2, 14), the same 1,024-token window in smaller
    blocks, and b = 32, b = 256;
  * a window without sinks.

Every window makes some key tiles partial for some rows (the sink tile, the
first local tile, the diagonal), which the b = 128 window never does. Tolerances
as everywhere: O max-abs 1e-2, mean-abs 1e-3; LSE max-abs 1e-3.
"""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, from_dev, to_dev

pytestmark = pytest.mark.gpu

WINDOWS = [(1, 16, 1024), (64, 2, 14), (32, 3, 20), (256, 1, 3), (1, 0, 300)]
IDS = ["tokens-16-1024", "b64-2-14", "b32-3-20", "b256-1-3", "tokens-0-300"]


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def prefill_case(bss, oracle_mod, seed, lens, H, Hkv, dqk, dv, scale, win, latent=False, workspace=True,
                 rows=None, what=""):
    import torch
    b, s, l = win
    g = synth.rng(seed)
    T = int(sum(lens))
    cu = synth.cu_seqlens(lens)
    q = synth.normal_bits(g, (T, H, dqk))
    if latent:
        kv = synth.normal_bits(g, (T, 1, dqk))
        k_bits, v_bits = kv, np.ascontiguousarray(kv[:, :, :dv])
        k_dev = to_dev(kv)
        v_dev = k_dev[:, :, :dv]
    else:
        k_bits = synth.normal_bits(g, (T, Hkv, dqk))
        v_bits = synth.normal_bits(g, (T, Hkv, dv))
        k_dev, v_dev = to_dev(k_bits), to_dev(v_bits)
    params = bss.Params(scale, b, s, l)
    ws = None
    if latent and workspace:
        n = bss.workspace_size(bss.LOZA_OP_PREFILL, len(lens), T, max(lens), H, Hkv, dqk, dv, params)
        assert n > 0, "the two-pass absorbed kernel takes this window"
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    elif latent:
        ws = torch.empty(16, dtype=torch.uint8, device="cuda")  # too small: the one-pass pair kernel
    out, lse = bss.loza_ssa_prefill(to_dev(q), k_dev, v_dev, torch.from_numpy(cu).cuda(), max(lens), params,
                                    workspace=ws)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.forward(q, k_bits, v_bits, cu, H, Hkv, b, s, l, scale, rows=rows)
    o_got, lse_got = from_dev(out), lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        o_got, lse_got = o_got[rows], lse_got[rows]
    assert_close_o(o_got, o_ref, f"{what} O {win}")
    assert_close_lse(lse_got, lse_ref, f"{what} LSE {win}")


@pytest.mark.parametrize("win", WINDOWS, ids=IDS)
def test_mha_d64_windows(bss, oracle_mod, win):
    """Workload 1's shapes (2,048 tokens, 4 heads, head dim 64, scale 1/8) and a
    packed batch with a 1-token and a ragged sequence."""
    prefill_case(bss, oracle_mod, synth.workload_seed(1), [2048], 4, 4, 64, 64, 1 / 8, win, what="cfg1")
    prefill_case(bss, oracle_mod, 601, [1000, 1, 2500], 2, 2, 64, 64, 1 / 8, win, what="mha packed")


@pytest.mark.parametrize("win", WINDOWS[:3], ids=IDS[:3])
def test_192_128_windows(bss, oracle_mod, win):
    prefill_case(bss, oracle_mod, 602, [2100, 700, 1], 2, 2, 192, 128, 1 / math.sqrt(192), win, what="192/128")


@pytest.mark.parametrize("workspace", [True, False], ids=["two-pass", "pair"])
@pytest.mark.parametrize("win", WINDOWS, ids=IDS)
def test_absorbed_windows(bss, oracle_mod, win, workspace):
    """Absorbed MLA (latent 576, V its first 512 columns) on a packed batch: the
    two-pass kernel (workspace given) and the one-pass CTA-pair kernel."""
    prefill_case(bss, oracle_mod, 603, [3000, 129, 1500], 8, 1, 576, 512, 1 / math.sqrt(192), win, latent=True,
                 workspace=workspace, what="absorbed")


@pytest.mark.parametrize("win", [(1, 16, 1024), (64, 2, 14)], ids=["tokens-16-1024", "b64-2-14"])
def test_absorbed_window_full_length(bss, oracle_mod, win):
    """Workload 2's shapes (L = 32,768, 64 heads, latent 576, scale 1/sqrt(192))
    under the window, through the two-pass kernel as bench.py runs it; sampled
    rows against the oracle."""
    import torch
    b, s, l = win
    L, H, D, DV = 32768, 64, 576, 512
    dev = torch.device("cuda")
    seed = synth.workload_seed(2) * 1000 + 11
    q = synth.torch_normal_bf16((L, H, D), seed, dev)
    lat = synth.torch_normal_bf16((L, 1, D), seed + 1, dev)
    cu = torch.tensor([0, L], dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(192.0)
    params = bss.Params(scale, b, s, l)
    ws = torch.empty(bss.workspace_size(bss.LOZA_OP_PREFILL, 1, L, L, H, 1, D, DV, params), dtype=torch.uint8,
                     device=dev)
    out, lse = bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], cu, L, params, workspace=ws)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    rs = np.random.default_rng(17)
    rows = np.unique(np.concatenate([[0, 15, 16, 17, 127, 128, 1023, 1024, 1025, 1100, 4095, L - 1],
                                     rs.choice(L, 40, replace=False)])).astype(np.int64)
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    q_host = np.empty((L, H, D), np.uint16)
    q_host[rows] = bits(q[torch.from_numpy(rows).to(dev)])
    lat_host = bits(lat)
    o_ref, lse_ref = oracle_mod.forward(q_host, lat_host, np.ascontiguousarray(lat_host[:, :, :DV]),
                                        synth.cu_seqlens([L]), H, 1, b, s, l, scale, rows=rows)
    idx = torch.from_numpy(rows).to(dev)
    assert_close_o(from_dev(out[idx]), o_ref, f"absorbed L=32768 O {win}")
    assert_close_lse(lse[idx].cpu().numpy().astype(np.float64), lse_ref, f"absorbed L=32768 LSE {win}")


def window_tile_rows(L, win, tile=128):
    """Rows of the 128-row tiles holding at least one key the decode query
    (position L - 1) sees: what the decode kernels may read."""
    b, s, l = win
    i = L - 1
    lo = max(0, (i // b - l + 1) * b)
    keys = np.concatenate([np.arange(0, min(s * b, L)), np.arange(max(lo, 0), L)])
    tiles = np.unique(keys // tile)
    return np.concatenate([np.arange(t * tile, min((t + 1) * tile, L)) for t in tiles])


def absorbed_decode_case(bss, oracle_mod, seed, lens, Lcap, win, poison=True):
    """Absorbed decode, 64 heads, latent cache [B, Lcap, 1, 576]: rows of the
    tiles the window reads carry seeded values (finite: they are context), every
    other row NaN (or zero)."""
    import torch
    H, D = 64, 576
    b, s, l = win
    B = len(lens)
    g = synth.rng(seed)
    q = synth.normal_bits(g, (B, H, D))
    cache_dev = torch.full((B, Lcap, 1, D), float("nan") if poison else 0.0, dtype=torch.bfloat16, device="cuda")
    host = np.empty((B, Lcap, 1, D), np.uint16)
    for n, L in enumerate(lens):
        rows = window_tile_rows(L, win)
        vals = synth.normal_bits(g, (len(rows), 1, D))
        host[n, rows] = vals
        cache_dev[n, torch.from_numpy(rows).cuda()] = to_dev(vals)
    seqlens = np.array(lens, np.int32)
    scale = 1.0 / math.sqrt(192.0)
    params = bss.Params(scale, b, s, l)
    out, lse = bss.loza_ssa_decode(to_dev(q), cache_dev, None, torch.from_numpy(seqlens).cuda(), Lcap, params)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.decode(q, host, None, seqlens, H, 1, b, s, l, scale, d_v=512)
    assert_close_o(from_dev(out), o_ref, f"absorbed decode O {win}")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, f"absorbed decode LSE {win}")
    res = (out.clone(), lse.clone())
    del cache_dev
    return res


@pytest.mark.parametrize("batch", [6, 40, 90], ids=["hb-4-splits", "hb-2-splits", "block-kernel"])
@pytest.mark.parametrize("win", WINDOWS, ids=IDS)
def test_absorbed_decode_windows(bss, oracle_mod, win, batch):
    """The decode plans: half blocks split over clusters of 4 (6 sequences) or 2
    (40), and the block kernel with one CTA per sequence (90); contexts from 1
    token to past the window, some on tile and half-tile edges."""
    g = synth.rng(700 + batch)
    lens = g.integers(1, 6000, size=batch)
    lens[:6] = [1, 17, 64, 1025, 1089, 5000]
    absorbed_decode_case(bss, oracle_mod, 701 + batch, lens.tolist(), 6144, win)


def test_absorbed_decode_window_nan_bitwise(bss, oracle_mod):
    """Rows outside the tiles the window reads are NaN: the output is finite
    and equals the zero-filled run bit for bit."""
    import torch
    for win in [(1, 16, 1024), (64, 2, 14)]:
        lens = [5, 300, 2049, 4000]
        o1, l1 = absorbed_decode_case(bss, oracle_mod, 720, lens, 4096, win, poison=True)
        o2, l2 = absorbed_decode_case(bss, oracle_mod, 720, lens, 4096, win, poison=False)
        assert torch.isfinite(o1.float()).all()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("win", [(1, 16, 1024), (64, 2, 14)], ids=["tokens-16-1024", "b64-2-14"])
def test_mha_decode_windows_and_prefill_row(bss, oracle_mod, win):
    """Per-head decode (workload 1's shapes: the last of 2,048 tokens, 4 heads,
    d = 64) against the oracle, and equal to the last row of the prefill."""
    import torch
    b, s, l = win
    H, dqk = 4, 64
    lens = [2048, 900, 1]
    B, Lcap = len(lens), max(lens)
    g = synth.rng(730)
    kc = synth.normal_bits(g, (B, Lcap, H, dqk))
    vc = synth.normal_bits(g, (B, Lcap, H, dqk))
    qd = synth.normal_bits(g, (B, H, dqk))
    params = bss.Params(1 / 8, b, s, l)
    seqlens = np.array(lens, np.int32)
    out, lse = bss.loza_ssa_decode(to_dev(qd), to_dev(kc), to_dev(vc), torch.from_numpy(seqlens).cuda(), Lcap,
                                   params)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.decode(qd, kc, vc, seqlens, H, H, b, s, l, 1 / 8)
    assert_close_o(from_dev(out), o_ref, f"mha decode O {win}")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, f"mha decode LSE {win}")
    for n, L in enumerate(lens):
        q = np.zeros((L, H, dqk), np.uint16)
        q[L - 1] = qd[n]
        cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
        po, pl = bss.loza_ssa_prefill(to_dev(q), to_dev(kc[n, :L]), to_dev(vc[n, :L]), cu, L, params)
        torch.cuda.synchronize()
        assert_close_o(from_dev(po[L - 1]), from_dev(out[n]), f"mha decode vs prefill row {win}")


@pytest.mark.parametrize("win", [(1, 16, 1024), (64, 2, 14)], ids=["tokens-16-1024", "b64-2-14"])
def test_absorbed_decode_equals_last_prefill_row_windows(bss, win):
    """Absorbed decode of the last token equals the last prefill row (576/512)
    under the window."""
    import torch
    b, s, l = win
    H, D, DV = 64, 576, 512
    lens = [1, 17, 1100, 5000]
    g = synth.rng(740)
    B, Lcap = len(lens), max(lens)
    qd = synth.normal_bits(g, (B, H, D))
    cache = torch.zeros((B, Lcap, 1, D), dtype=torch.bfloat16, device="cuda")
    for n, L in enumerate(lens):
        cache[n, :L] = to_dev(synth.normal_bits(g, (L, 1, D)))
    params = bss.Params(1.0 / math.sqrt(192.0), b, s, l)
    out, lse = bss.loza_ssa_decode(to_dev(qd), cache, None, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                   Lcap, params)
    torch.cuda.synchronize()
    for n, L in enumerate(lens):
        q = torch.zeros((L, H, D), dtype=torch.bfloat16, device="cuda")
        q[L - 1] = to_dev(qd[n])
        lat = cache[n, :L].contiguous()
        po, pl = bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], torch.tensor([0, L], dtype=torch.int32, device="cuda"),
                                      L, params)
        torch.cuda.synchronize()
        assert_close_o(from_dev(po[L - 1]), from_dev(out[n]), f"absorbed decode vs prefill row {win} L={L}")
        assert_close_lse(pl[L - 1].cpu().numpy().astype(np.float64), lse[n].cpu().numpy().astype(np.float64),
                         f"absorbed decode vs prefill row LSE {win} L={L}")
