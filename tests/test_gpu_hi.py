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
    """Index queries and keys: N(0, 1) in bf16; small integers (ints=True:
    exact scores, many ties); or 0/1 keys against an all-ones query
    (ints="binary": scores crowd into a few values)."""
    if ints == "binary":
        ones = np.full((B, d), 0x3F80, np.uint16)
        return ones, synth.bf16_bits(g.integers(0, 2, size=(B, Lcap, d)).astype(np.float32))
    if ints:
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
    ref = oracle_mod.hi_page_keys(k_idx, lens)          # [B, pages, d]; the library's is [B, d, pages]
    for n, L in enumerate(lens):
        np.testing.assert_array_equal(pk[n, :, :L // 128].T, ref[n, :L // 128])


SELECT_CASES = [
    # (window, top_pages, top_k, d, integer keys)
    (TOKEN_WINDOW, 8, 500, 64, False),
    (TOKEN_WINDOW, 1024, 1024, 128, False),   # page 4's budget: 1,024 pages and 1,024 tokens
    ((128, 1, 7), 64, 2048, 64, False),       # the SSA block window; the largest top_k
    ((64, 2, 3), 3, 100, 192, False),         # fewer tokens kept than the pages hold
    ((1, 0, 50), 10 ** 4, 7, 64, False),      # more pages asked than exist
    (TOKEN_WINDOW, 6, 300, 64, True),         # many equal scores: ties go to the lower index
    (TOKEN_WINDOW, 150, 2000, 64, "binary"),  # more than 4,096 keys share the threshold's top digit
    ((128, 1, 7), 40, 1500, 512, False),      # the widest index key
]


@pytest.mark.parametrize("win,top_pages,top_k,d,ints", SELECT_CASES,
                         ids=[f"w{c[0][0]}-{c[0][1]}-{c[0][2]}-p{c[1]}-k{c[2]}-d{c[3]}{'-' + str(c[4]) if c[4] else ''}"
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
    q_idx, k_idx = index_inputs(g, 2, 5000, 64)
    _, sel = gpu_select(bss, q_idx, k_idx, lens, 5000, (128, 1, -1), 4, 64)
    assert (sel == -1).all()


def filled_cache(g, lens, Lcap, win, extra_rows, poison=True):
    """Latent cache [B, Lcap, 1, 576]: the rows of the tiles the window reads
    and the rows in extra_rows[n] carry seeded values, every other row is NaN
    (or zero); returns the device cache and its host copy."""
    import torch
    B = len(lens)
    cache = torch.full((B, Lcap, 1, D), float("nan") if poison else 0.0, dtype=torch.bfloat16, device="cuda")
    host = np.empty((B, Lcap, 1, D), np.uint16)
    for n, L in enumerate(lens):
        rows = np.union1d(window_tile_rows(L, win), extra_rows[n])
        vals = synth.normal_bits(g, (len(rows), 1, D))
        host[n, rows] = vals
        cache[n, torch.from_numpy(rows).cuda()] = to_dev(vals)
    return cache, host


def attention_case(bss, oracle_mod, seed, lens, Lcap, win, top_pages, top_k, d_index=64, poison=True):
    """The whole decode on the GPU against the oracle, and the same selection
    through loza_ssa_decode_selected."""
    import torch
    B = len(lens)
    g = synth.rng(seed)
    q_idx, k_idx = index_inputs(g, B, Lcap, d_index)
    ref_sel = oracle_mod.hi_select(q_idx, k_idx, oracle_mod.hi_page_keys(k_idx, lens), lens, *win, top_pages,
                                   top_k)
    q = synth.normal_bits(g, (B, H, D))
    cache, host = filled_cache(g, lens, Lcap, win, [r[r >= 0] for r in ref_sel], poison)
    scale = 1.0 / math.sqrt(192.0)
    p = bss.Params(scale, *win)
    seq = dev_i32(lens)
    k_dev = to_dev(k_idx)
    pk = bss.loza_hi_page_keys(k_dev, seq, Lcap)
    q_dev = to_dev(q)
    out, lse = bss.loza_hi_decode(q_dev, cache, to_dev(q_idx), k_dev, pk, seq, Lcap, p, top_pages, top_k)
    o_s, l_s = bss.loza_ssa_decode_selected(q_dev, cache, seq, Lcap, p, dev_i32(ref_sel))
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.hi_decode(q, host, lens, H, *win, scale, ref_sel)
    tag = f"{win} p{top_pages} k{top_k}"
    assert_close_o(from_dev(out), o_ref, f"HI decode O {tag}")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, f"HI decode LSE {tag}")
    # the same computation from the oracle's selection: bit for bit the same
    assert torch.equal(out, o_s) and torch.equal(lse, l_s)
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


def test_decode_selected_with_a_caller_list(bss, oracle_mod):
    """A caller's own list: unsorted, with -1 holes and entries that the call
    must ignore (inside the window, past the query); the rest is attended with
    the window."""
    import torch
    g = synth.rng(935)
    lens, Lcap, win = [6000, 3000, 1200, 40], 6144, TOKEN_WINDOW
    B, top_k = len(lens), 700
    lists = np.full((B, top_k), -1, np.int32)
    kept = []
    for n, L in enumerate(lens):
        outside = np.array([t for t in range(L) if t >= 16 and t < max(0, L - 1024)], np.int64)
        take = g.choice(outside, size=min(len(outside), 500), replace=False) if len(outside) else outside
        ignored = np.concatenate([np.arange(0, min(16, L)), np.arange(max(0, L - 5), L), L + np.arange(3)])
        entries = np.concatenate([take, ignored])
        slots = g.choice(top_k, size=len(entries), replace=False)
        lists[n, slots] = entries
        kept.append(np.sort(take).astype(np.int32))
    q = synth.normal_bits(g, (B, H, D))
    cache, host = filled_cache(g, lens, Lcap, win, kept)
    scale = 1.0 / math.sqrt(192.0)
    out, lse = bss.loza_ssa_decode_selected(to_dev(q), cache, dev_i32(lens), Lcap, bss.Params(scale, *win),
                                            dev_i32(lists))
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    ref_list = np.full((B, top_k), -1, np.int32)
    for n, k in enumerate(kept):
        ref_list[n, :len(k)] = k
    o_ref, lse_ref = oracle_mod.hi_decode(q, host, lens, H, *win, scale, ref_list)
    assert_close_o(from_dev(out), o_ref, "decode over a caller list O")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "decode over a caller list LSE")


def test_hi_decode_unbounded_window_is_full_attention(bss, oracle_mod):
    import torch
    g = synth.rng(936)
    lens, Lcap = [3000, 129, 1], 3072
    B = len(lens)
    q_idx, k_idx = index_inputs(g, B, Lcap, 64)
    q = synth.normal_bits(g, (B, H, D))
    kv = synth.normal_bits(g, (B, Lcap, 1, D))
    scale = 1.0 / math.sqrt(192.0)
    seq = dev_i32(lens)
    k_dev = to_dev(k_idx)
    pk = bss.loza_hi_page_keys(k_dev, seq, Lcap)
    out, lse = bss.loza_hi_decode(to_dev(q), to_dev(kv), to_dev(q_idx), k_dev, pk, seq, Lcap,
                                  bss.Params(scale, 128, 1, -1), 8, 256)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.decode(q, kv, None, np.array(lens, np.int32), H, 1, 128, 0, -1, scale, d_v=512)
    assert_close_o(from_dev(out), o_ref, "HI decode, unbounded window O")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "HI decode, unbounded window LSE")


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
    pk_h = pk.cpu().numpy()
    np.testing.assert_array_equal(pk_h[0].T, pk_ref[0])
    np.testing.assert_array_equal(pk_h[1, :, :lens[1] // 128].T, pk_ref[1, :lens[1] // 128])
    ref_sel = oracle_mod.hi_select(q_idx, k_idx, pk_ref, lens, *TOKEN_WINDOW, top_pages, top_k)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    # the decode over window and selection, with every other cache row NaN
    q = synth.normal_bits(g, (B, H, D))
    cache, host = filled_cache(g, lens, Lcap, TOKEN_WINDOW, [r[r >= 0] for r in ref_sel])
    scale = 1.0 / math.sqrt(192.0)
    out, lse = bss.loza_hi_decode(to_dev(q), cache, to_dev(q_idx), k_dev, pk, seq, Lcap,
                                  bss.Params(scale, *TOKEN_WINDOW), top_pages, top_k)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.hi_decode(q, host, lens, H, *TOKEN_WINDOW, scale, ref_sel)
    assert_close_o(from_dev(out), o_ref, "HI decode 1M O")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "HI decode 1M LSE")
