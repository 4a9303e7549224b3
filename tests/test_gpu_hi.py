"""GPU parity of the hierarchical index decode against the oracle (page 4,
"LongCat Sparse Attention": pages of 128 tokens scored by a coarse pass, the
top pages recalled, their tokens scored one by one and the best kept; the
fixed sink and window part and the dynamic part attended apart and merged by
their log-sum-exp).

The page keys and the selection are integer and index work decided by fp32
scores that both sides form in the same order, so they must match bit for bit.
The attention is compared within the O / LSE tolerances. Cache rows that are
neither in a tile the window reads nor selected are NaN, so a read outside the
selection shows up as a non-finite or wrong output."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, from_dev, to_dev

pytestmark = pytest.mark.gpu

H, D = 64, 576
TOKEN_WINDOW = (1, 16, 1024)   # page 4: 16 sink tokens and a 1,024-token window


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def window_tile_rows(L, win, tile=128):
    """Rows of the 128-row tiles holding a key of the window of the decode
    query (position L - 1): what the window decode may read."""
    b, s, l = win
    i = L - 1
    if l < 0:
        return np.arange(L)
    lo = max(0, (i // b - l + 1) * b)
    keys = np.concatenate([np.arange(0, min(s * b, L)), np.arange(lo, L)])
    tiles = np.unique(keys // tile)
    return np.concatenate([np.arange(t * tile, min((t + 1) * tile, L)) for t in tiles])


def index_inputs(g, B, Lcap, d, ints=False):
    if ints:  # small integers: exact scores with many ties
        draw = lambda shape: synth.bf16_bits(g.integers(-3, 4, size=shape).astype(np.float32))
    else:
        draw = lambda shape: synth.normal_bits(g, shape)
    return draw((B, d)), draw((B, Lcap, d))


def gpu_select(bss, q_idx, k_idx, lens, Lcap, win, top_pages, top_k, k_dev=None):
    import torch
    k_dev = to_dev(k_idx) if k_dev is None else k_dev
    seq = dev_i32(lens)
    pk = bss.loza_hi_page_keys(k_dev, seq, Lcap)
    p = bss.Params(0.1, *win)
    sel = bss.loza_hi_select(to_dev(q_idx), k_dev, pk, seq, Lcap, p, top_pages, top_k)
    torch.cuda.synchronize()
    return pk.cpu().numpy(), sel.cpu().numpy()


def test_page_keys_bit_exact(bss, oracle_mod):
    g = synth.rng(901)
    lens = [5000, 129, 100, 128, 4096]
    q_idx, k_idx = index_inputs(g, len(lens), 5120, 64)
    pk, _ = gpu_select(bss, q_idx, k_idx, lens, 5120, TOKEN_WINDOW, 4, 16)
    ref = oracle_mod.hi_page_keys(k_idx, lens)
    for n, L in enumerate(lens):
        np.testing.assert_array_equal(pk[n, :L // 128], ref[n, :L // 128])


SELECT_CASES = [
    # (window, top_pages, top_k, d, integer keys)
    (TOKEN_WINDOW, 8, 500, 64, False),
    (TOKEN_WINDOW, 1024, 1024, 128, False),   # page 4's budget: 1,024 pages and 1,024 tokens
    ((128, 1, 7), 64, 2048, 32, False),       # the SSA block window; the largest top_k
    ((64, 2, 3), 3, 100, 8, False),           # fewer tokens kept than the pages hold
    ((1, 0, 50), 10 ** 4, 7, 16, False),      # more pages asked than exist
    (TOKEN_WINDOW, 6, 300, 16, True),         # many equal scores: ties go to the lower index
    ((128, 1, 7), 40, 1500, 512, False),      # the widest index key
]


@pytest.mark.parametrize("win,top_pages,top_k,d,ints", SELECT_CASES,
                         ids=[f"w{c[0][0]}-{c[0][1]}-{c[0][2]}-p{c[1]}-k{c[2]}-d{c[3]}{'-int' if c[4] else ''}"
                              for c in SELECT_CASES])
def test_selection_is_the_oracles(bss, oracle_mod, win, top_pages, top_k, d, ints):
    g = synth.rng(910 + top_k + d)
    lens = [1, 127, 1200, 1152, 5000, 20000, 20480, 9001]
    Lcap = 20480
    q_idx, k_idx = index_inputs(g, len(lens), Lcap, d, ints)
    _, sel = gpu_select(bss, q_idx, k_idx, lens, Lcap, win, top_pages, top_k)
    ref = oracle_mod.hi_select(q_idx, k_idx, oracle_mod.hi_page_keys(k_idx, lens), lens, *win, top_pages, top_k)
    np.testing.assert_array_equal(sel, ref)


def test_selection_with_strided_index_rows(bss, oracle_mod):
    """Index keys stored inside wider rows (row stride 2d) and a batch stride
    beyond the rows used."""
    import torch
    g = synth.rng(920)
    lens, Lcap, d = [3000, 700, 4096], 4096, 64
    q_idx, k_idx = index_inputs(g, len(lens), Lcap, d)
    wide = torch.zeros((len(lens), Lcap + 64, 2 * d), dtype=torch.bfloat16, device="cuda")
    wide[:, :Lcap, :d] = to_dev(k_idx)
    _, sel = gpu_select(bss, q_idx, k_idx, lens, Lcap, TOKEN_WINDOW, 5, 333, k_dev=wide[:, :Lcap, :d])
    ref = oracle_mod.hi_select(q_idx, k_idx, oracle_mod.hi_page_keys(k_idx, lens), lens, *TOKEN_WINDOW, 5, 333)
    np.testing.assert_array_equal(sel, ref)


def test_unbounded_window_selects_nothing(bss):
    """With full causal attention as the window no token lies outside it."""
    g = synth.rng(921)
    lens = [5000, 300]
    q_idx, k_idx = index_inputs(g, 2, 5000, 32)
    _, sel = gpu_select(bss, q_idx, k_idx, lens, 5000, (128, 1, -1), 4, 64)
    assert (sel == -1).all()


def attention_case(bss, oracle_mod, seed, lens, Lcap, win, top_pages, top_k, d_index=64, poison=True):
    """The whole decode on the GPU against the oracle; also the two parts apart
    (the selected part through loza_ssa_decode_selected)."""
    import torch
    B = len(lens)
    g = synth.rng(seed)
    q_idx, k_idx = index_inputs(g, B, Lcap, d_index)
    ref_sel = oracle_mod.hi_select(q_idx, k_idx, oracle_mod.hi_page_keys(k_idx, lens), lens, *win, top_pages,
                                   top_k)
    q = synth.normal_bits(g, (B, H, D))
    cache = torch.full((B, Lcap, 1, D), float("nan") if poison else 0.0, dtype=torch.bfloat16, device="cuda")
    host = np.empty((B, Lcap, 1, D), np.uint16)
    for n, L in enumerate(lens):
        rows = np.union1d(window_tile_rows(L, win), ref_sel[n][ref_sel[n] >= 0])
        vals = synth.normal_bits(g, (len(rows), 1, D))
        host[n, rows] = vals
        cache[n, torch.from_numpy(rows).cuda()] = to_dev(vals)
    scale = 1.0 / math.sqrt(192.0)
    p = bss.Params(scale, *win)
    seq = dev_i32(lens)
    k_dev = to_dev(k_idx)
    pk = bss.loza_hi_page_keys(k_dev, seq, Lcap)
    q_dev = to_dev(q)
    out, lse = bss.loza_hi_decode(q_dev, cache, to_dev(q_idx), k_dev, pk, seq, Lcap, p, top_pages, top_k)
    # the selected part alone, from the oracle's selection
    o_s, l_s = bss.loza_ssa_decode_selected(q_dev, cache, dev_i32(ref_sel), scale)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.hi_decode(q, host, lens, H, *win, scale, ref_sel)
    assert_close_o(from_dev(out), o_ref, f"HI decode O {win} p{top_pages} k{top_k}")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, f"HI decode LSE {win} p{top_pages} k{top_k}")
    # an empty window (no sinks, no local keys) leaves the selection alone
    has = (ref_sel >= 0).any(axis=1)
    o_sr, l_sr = oracle_mod.hi_decode(q[has], host[has], np.asarray(lens)[has], H, 1, 0, 0, scale, ref_sel[has])
    assert_close_o(from_dev(o_s)[has], o_sr, f"selected part O {win}")
    assert_close_lse(l_s.cpu().numpy().astype(np.float64)[has], l_sr, f"selected part LSE {win}")
    empty_l = l_s.cpu().numpy()[~has]
    assert np.all(empty_l == -np.inf) and not from_dev(o_s)[~has].any()
    res = (out.clone(), lse.clone())
    del cache
    return res


@pytest.mark.parametrize("win", [TOKEN_WINDOW, (128, 1, 7), (64, 2, 14)], ids=["tokens-16-1024", "b128-1-7",
                                                                             "b64-2-14"])
def test_hi_decode(bss, oracle_mod, win):
    lens = [1, 200, 1100, 1500, 3000, 8192, 12000, 7]
    attention_case(bss, oracle_mod, 930, lens, 12288, win, 16, 1024)


def test_hi_decode_batches_and_budgets(bss, oracle_mod):
    """A larger batch (the window decode takes its other plans) with a small
    budget, and one sequence with a full budget of page 4's size."""
    g = synth.rng(931)
    lens = g.integers(1, 9000, size=40).tolist()
    attention_case(bss, oracle_mod, 932, lens, 9216, TOKEN_WINDOW, 4, 64)
    attention_case(bss, oracle_mod, 933, [40000], 40960, TOKEN_WINDOW, 1024, 1024)


def test_hi_decode_nan_bounds_bitwise(bss, oracle_mod):
    """Rows neither read by the window nor selected are NaN: the output is
    finite and equals the zero-filled run bit for bit."""
    import torch
    lens = [2500, 5000, 333]
    o1, l1 = attention_case(bss, oracle_mod, 940, lens, 5120, TOKEN_WINDOW, 8, 512, poison=True)
    o2, l2 = attention_case(bss, oracle_mod, 940, lens, 5120, TOKEN_WINDOW, 8, 512, poison=False)
    assert torch.isfinite(o1.float()).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_hi_decode_one_million_tokens(bss, oracle_mod):
    """Two sequences of 1,048,576 and 700,001 tokens (8,192 pages, the most the
    page sort holds), page 4's budget: 16 sink tokens, a 1,024-token window,
    1,024 recalled pages and 1,024 selected tokens. Index keys are drawn on the
    device (seeded) and copied to the host for the oracle."""
    import torch
    Lcap, d = 1 << 20, 64
    lens = [Lcap, 700001]
    B = len(lens)
    k_dev = synth.torch_normal_bf16((B, Lcap, d), 950, "cuda")
    k_idx = k_dev.view(torch.int16).cpu().numpy().view(np.uint16)
    g = synth.rng(951)
    q_idx = synth.normal_bits(g, (B, d))
    top_pages, top_k = 1024, 1024
    seq = dev_i32(lens)
    pk = bss.loza_hi_page_keys(k_dev, seq, Lcap)
    sel = bss.loza_hi_select(to_dev(q_idx), k_dev, pk, seq, Lcap, bss.Params(0.1, *TOKEN_WINDOW), top_pages, top_k)
    torch.cuda.synchronize()
    pk_ref = oracle_mod.hi_page_keys(k_idx, lens)
    np.testing.assert_array_equal(pk.cpu().numpy()[0], pk_ref[0])
    np.testing.assert_array_equal(pk.cpu().numpy()[1, :lens[1] // 128], pk_ref[1, :lens[1] // 128])
    ref_sel = oracle_mod.hi_select(q_idx, k_idx, pk_ref, lens, *TOKEN_WINDOW, top_pages, top_k)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    # the decode over window and selection, with every other cache row NaN
    q = synth.normal_bits(g, (B, H, D))
    cache = torch.full((B, Lcap, 1, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    host = np.empty((B, Lcap, 1, D), np.uint16)
    for n, L in enumerate(lens):
        rows = np.union1d(window_tile_rows(L, TOKEN_WINDOW), ref_sel[n][ref_sel[n] >= 0])
        vals = synth.normal_bits(g, (len(rows), 1, D))
        host[n, rows] = vals
        cache[n, torch.from_numpy(rows).cuda()] = to_dev(vals)
    scale = 1.0 / math.sqrt(192.0)
    out, lse = bss.loza_hi_decode(to_dev(q), cache, to_dev(q_idx), k_dev, pk, seq, Lcap,
                                  bss.Params(scale, *TOKEN_WINDOW), top_pages, top_k)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.hi_decode(q, host, lens, H, *TOKEN_WINDOW, scale, ref_sel)
    assert_close_o(from_dev(out), o_ref, "HI decode 1M O")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "HI decode 1M LSE")
