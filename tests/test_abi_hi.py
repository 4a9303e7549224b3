"""Host-side checks of the hierarchical index entry points (page 4's
streaming-aware, hierarchical index: pages of 128 tokens, top pages, then top
tokens): argument validation before any launch, and the workspace size. No
GPU: every call here is rejected on the host, or only sizes a buffer."""
import ctypes

import pytest

import block_sparse_streaming_b200 as bss

vp = ctypes.c_void_p
OK, INVALID, UNSUPPORTED, WORKSPACE = 0, -1, -2, -3


@pytest.fixture(scope="module")
def L():
    bss.build()
    return bss.lib()


def _index(**over):
    a = dict(k=1 << 21, bs=4096 * 64, rs=64, seqlens=1 << 22, batch=2, max_seqlen=4096, d=64)
    a.update(over)
    return a


@pytest.mark.parametrize("over", [
    dict(k=0), dict(k=(1 << 21) + 8),          # null / misaligned index keys
    dict(seqlens=0),
    dict(d=12, rs=12, bs=4096 * 12),            # d_index not a multiple of 64
    dict(d=32, rs=32, bs=4096 * 32),
    dict(d=520, rs=520, bs=4096 * 520),         # d_index above 512
    dict(d=0),
    dict(rs=32),                                # row stride below d_index
    dict(rs=68, bs=4096 * 68),                  # row stride not 16-byte
    dict(bs=4095 * 64),                         # batch stride below max_seqlen rows
    dict(batch=0), dict(max_seqlen=0),
])
def test_page_keys_rejects_before_launch(L, over):
    a = _index(**over)
    count = L.loza_launch_count()
    rc = L.loza_hi_page_keys(vp(a["k"]), a["bs"], a["rs"], vp(a["seqlens"]), a["batch"], a["max_seqlen"], a["d"],
                             vp(1 << 23), vp(0))
    assert rc == INVALID
    assert L.loza_launch_count() == count


def test_workspace_size():
    p = bss.Params(0.07, block_size=1, n_sink=16, n_local=1024)
    size = bss.hi_workspace_size
    base = size(4, 1 << 20, 1024, 1024, p)
    assert base > 0 and base % 256 == 0
    assert size(4, 1 << 20, 2048, 1024, p) > base    # the token keys grow with the recalled pages
    assert size(8, 1 << 20, 1024, 1024, p) > base    # and everything with the batch
    assert size(4, 1 << 20, 1024, 2048, p) >= base
    assert size(4, 1 << 20, 1024, 2049, p) == 0      # top_k above 2,048
    assert size(4, 1 << 20, 0, 1024, p) == 0         # no page recalled
    assert size(0, 1 << 20, 1024, 1024, p) == 0
    assert size(4, 1 << 20, 1024, 1024, bss.Params(0.07, block_size=3)) == 0
    assert size(4, 1 << 20, 1024, 1024, bss.Params(0.07, block_size=128, n_sink=1, n_local=512)) == 0  # window > 64K rows
    assert size(4, 1 << 20, 1024, 1024, bss.Params(0.07, block_size=128, n_sink=1, n_local=-1)) > 0   # unbounded


def _select(L, ws_bytes=1 << 30, ws=1 << 24, top_pages=16, top_k=256, params=None, q_index=1 << 20, **over):
    a = _index(**over)
    p = params or bss.Params(0.07, block_size=1, n_sink=16, n_local=1024)
    return L.loza_hi_select(vp(q_index), vp(a["k"]), a["bs"], a["rs"], vp(1 << 23), vp(a["seqlens"]), a["batch"],
                            a["max_seqlen"], a["d"], p, top_pages, top_k, vp(1 << 25), vp(ws), ws_bytes, vp(0))


@pytest.mark.parametrize("kw,code", [
    (dict(q_index=0), INVALID),
    (dict(q_index=(1 << 20) + 4), INVALID),
    (dict(top_k=0), INVALID),
    (dict(top_k=2049), INVALID),
    (dict(top_pages=0), INVALID),
    (dict(d=12, rs=12, bs=4096 * 12), INVALID),
    (dict(params=bss.Params(0.07, block_size=96)), UNSUPPORTED),
    (dict(max_seqlen=8193 * 128, bs=8193 * 128 * 64), UNSUPPORTED),  # more pages than the page sort holds
    (dict(ws=0), INVALID),
    (dict(ws=(1 << 24) + 128), INVALID),         # workspace not 256-byte aligned
    (dict(ws_bytes=1024), WORKSPACE),
])
def test_select_rejects_before_launch(L, kw, code):
    count = L.loza_launch_count()
    assert _select(L, **kw) == code
    assert L.loza_launch_count() == count


@pytest.mark.parametrize("q,kv,rs,top_k,sel,params,ws_bytes,code", [
    (0, 1 << 21, 576, 64, 1 << 22, None, 1 << 30, INVALID),
    (1 << 20, (1 << 21) + 2, 576, 64, 1 << 22, None, 1 << 30, INVALID),
    (1 << 20, 1 << 21, 512, 64, 1 << 22, None, 1 << 30, INVALID),     # latent row narrower than 576
    (1 << 20, 1 << 21, 580, 64, 1 << 22, None, 1 << 30, INVALID),     # row stride not 16-byte
    (1 << 20, 1 << 21, 576, -1, 1 << 22, None, 1 << 30, INVALID),
    (1 << 20, 1 << 21, 576, 2049, 1 << 22, None, 1 << 30, INVALID),
    (1 << 20, 1 << 21, 576, 64, 0, None, 1 << 30, INVALID),           # no list
    (1 << 20, 1 << 21, 576, 64, 1 << 22, bss.Params(0.07, block_size=6), 1 << 30, UNSUPPORTED),
    (0, 1 << 21, 576, 64, 1 << 22, None, 4096, WORKSPACE),  # q NULL: a skipped size check still launches nothing
])
def test_decode_selected_rejects_before_launch(L, q, kv, rs, top_k, sel, params, ws_bytes, code):
    p = params or bss.Params(0.07, block_size=1, n_sink=16, n_local=1024)
    count = L.loza_launch_count()
    rc = L.loza_ssa_decode_selected(vp(q), vp(kv), 4096 * rs, rs, vp(1 << 23), 2, 4096, p, vp(sel), top_k,
                                    vp(1 << 24), vp(1 << 25), vp(1 << 26), ws_bytes, vp(0))
    assert rc == code
    assert L.loza_launch_count() == count


def _hi_decode(L, ws_bytes=1 << 30, ws=1 << 26, q=1 << 27, cache_rs=576, top_k=256, params=None, **over):
    a = _index(**over)
    p = params or bss.Params(0.07, block_size=1, n_sink=16, n_local=1024)
    return L.loza_hi_decode(vp(q), vp(1 << 28), a["max_seqlen"] * cache_rs, cache_rs, vp(1 << 20), vp(a["k"]),
                            a["bs"], a["rs"], vp(1 << 23), vp(a["seqlens"]), a["batch"], a["max_seqlen"], a["d"], p,
                            16, top_k, vp(1 << 29), vp(1 << 30), vp(ws), ws_bytes, vp(0))


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), INVALID),
    (dict(cache_rs=512), INVALID),
    (dict(top_k=4096), INVALID),
    (dict(k=0), INVALID),
    (dict(params=bss.Params(0.07, block_size=5)), UNSUPPORTED),
    (dict(ws=0), INVALID),
    (dict(ws_bytes=4096, q=0), WORKSPACE),  # q NULL: a skipped size check still launches nothing
])
def test_hi_decode_rejects_before_launch(L, kw, code):
    count = L.loza_launch_count()
    assert _hi_decode(L, **kw) == code
    assert L.loza_launch_count() == count
