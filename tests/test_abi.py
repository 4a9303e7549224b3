"""Host-side checks of the C-ABI library that need no GPU: it builds, loads,
exports every symbol the header declares, and rejects bad arguments before
launching anything."""
import ctypes
import math
import os
import re

import pytest

import block_sparse_streaming_b200 as bss

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    bss.build()
    return bss.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "loza_ssa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(loza_[a-z_]+)\s*\(", src)))


def test_header_declares_binding_names():
    assert declared_functions() == sorted(bss.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5):
        assert L.loza_status_string(code)
    assert L.loza_status_string(42) == b"unknown status"


def _prefill_args(**over):
    a = dict(q=1 << 20, k=1 << 21, v=1 << 22, cu=1 << 23, batch=1, T=256, max_seqlen=256, H=4, Hkv=4,
             dqk=64, dv=64, qs=256, ks=256, vs=256, params=bss.Params(0.125), out=1 << 24, lse=1 << 25)
    a.update(over)
    return a


def _call_prefill(L, a):
    vp = ctypes.c_void_p
    return L.loza_ssa_prefill(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["cu"]), a["batch"], a["T"],
                              a["max_seqlen"], a["H"], a["Hkv"], a["dqk"], a["dv"], a["qs"], a["ks"], a["vs"],
                              a["params"], vp(a["out"]), vp(a["lse"]), vp(0), 0, vp(0))


@pytest.mark.parametrize("over,code", [
    (dict(q=0), -1),                       # null pointer
    (dict(q=(1 << 20) + 2), -1),           # misaligned
    (dict(H=6, Hkv=4), -1),                # heads not a multiple of kv heads
    (dict(qs=100), -1),                    # row stride below heads*dim
    (dict(qs=257), -1),                    # row stride not 16-byte
    (dict(batch=0), -1),
    (dict(max_seqlen=300), -1),            # longer than the packed batch
    (dict(dqk=96, dv=96, qs=384, ks=384, vs=384), -2),    # head dims not compiled
    (dict(params=bss.Params(0.1, block_size=96)), -2),    # b must be a power of two
    (dict(params=bss.Params(0.1, block_size=0)), -2),
    (dict(params=bss.Params(0.1, block_size=1 << 17)), -2),  # at most 65,536
    (dict(params=bss.Params(0.1, block_size=1 << 16, n_local=1 << 15)), -2),  # window beyond 2^30 keys
    (dict(params=bss.Params(0.1, n_local=0)), -2),
    (dict(H=4, Hkv=2, ks=128, vs=128), -2),              # grouped heads not compiled
])
def test_prefill_rejects_before_launch(L, over, code):
    count = L.loza_launch_count()
    assert _call_prefill(L, _prefill_args(**over)) == code
    assert L.loza_launch_count() == count


@pytest.mark.parametrize("rows,d_v,o_a,code", [
    (-1, 512, 1 << 20, -1),          # negative row count
    (4, 12, 1 << 20, -1),            # d_v not a multiple of 8
    (4, 0, 1 << 20, -1),
    (4, 512, 0, -1),                 # null branch
    (4, 512, (1 << 20) + 8, -1),     # misaligned branch
    (0, 512, 0, 0),                  # nothing to do: no launch, ok
])
def test_merge_rejects_before_launch(L, rows, d_v, o_a, code):
    vp = ctypes.c_void_p
    count = L.loza_launch_count()
    rc = L.loza_ssa_merge(vp(o_a), vp(1 << 21), vp(1 << 22), vp(1 << 23), rows, d_v, vp(1 << 24), vp(1 << 25),
                          vp(0))
    assert rc == code
    assert L.loza_launch_count() == count


@pytest.mark.parametrize("n,out,code", [(-8, 1 << 22, -1), (12, 1 << 22, -1), (16, 0, -1), (16, (1 << 22) + 4, -1),
                                        (0, 0, 0)])
def test_mix_rejects_before_launch(L, n, out, code):
    vp = ctypes.c_void_p
    count = L.loza_launch_count()
    assert L.loza_ssa_mix(vp(1 << 20), vp(1 << 21), n, 0.5, vp(out), vp(0)) == code
    assert L.loza_launch_count() == count


@pytest.mark.parametrize("table,bt_stride,num_pages,code", [
    (0, 8, 16, -1),              # no block table
    (1 << 26, 7, 16, -1),        # fewer table columns than blocks of max_seqlen (1024 -> 8)
    (1 << 26, 8, 0, -1),         # empty pool
    (1 << 26, 8, 1 << 24, -1),   # pool rows beyond int32
])
def test_decode_paged_rejects_before_launch(L, table, bt_stride, num_pages, code):
    vp = ctypes.c_void_p
    count = L.loza_launch_count()
    rc = L.loza_ssa_decode_paged(vp(1 << 20), vp(1 << 21), num_pages, 576, vp(table), bt_stride, vp(1 << 22), 4,
                                 1024, 64, bss.Params(1 / 8), vp(1 << 23), vp(1 << 24), vp(0), 0, vp(0))
    assert rc == code
    assert L.loza_launch_count() == count


def _call_prefill_host(L, q=1 << 20, k=1 << 21, v=1 << 22, cu=(0, 4096), batch=None, total=None, max_seqlen=None,
                       H=4, Hkv=4, dqk=64, dv=64, params=None, ws=1 << 28, ws_bytes=1 << 40, null_cu=False):
    import numpy as np
    vp = ctypes.c_void_p
    params = params if params is not None else bss.Params(0.125)
    cu_arr = np.ascontiguousarray(cu, dtype=np.int32)  # host memory, as the entry point requires
    batch = len(cu) - 1 if batch is None else batch
    total = int(cu[-1]) if total is None else total
    max_seqlen = int(max(np.diff(cu))) if max_seqlen is None else max_seqlen
    cu_ptr = vp(0) if null_cu else cu_arr.ctypes.data_as(vp)
    return L.loza_ssa_prefill_host(vp(q), vp(k), vp(v), cu_ptr, batch, total, max_seqlen, H, Hkv, dqk, dv, params,
                                   vp(1 << 24), vp(1 << 25), vp(ws), ws_bytes, vp(0))


@pytest.mark.parametrize("over,code", [
    (dict(q=0), -1),                                  # null pointer
    (dict(null_cu=True), -1),                         # no sequence offsets
    (dict(cu=(0, 0), max_seqlen=1), -1),              # no tokens at all
    (dict(cu=(0, 100, 50, 200)), -1),                 # offsets going backwards
    (dict(cu=(1, 100)), -1),                          # offsets not starting at 0
    (dict(cu=(0, 100, 300), max_seqlen=150), -1),     # a sequence longer than max_seqlen
    (dict(cu=(0, 100, 300), total=299), -1),          # last offset is not the token count
    (dict(H=6, Hkv=4), -1),                           # heads not a multiple of kv heads
    (dict(H=4, Hkv=2), -2),                           # grouped heads not compiled
    (dict(dqk=96, dv=96), -2),                        # head dims not compiled
    (dict(dqk=576, dv=512, H=3, Hkv=1), -2),          # absorbed needs an even head count
    (dict(params=bss.Params(0.1, n_local=0)), -2),    # empty local window
    (dict(params=bss.Params(0.1, 96, 1, 7)), -2),     # block size not a power of two
    (dict(ws=0), -1),                                 # no workspace
    (dict(ws=(1 << 28) + 16), -1),                    # workspace not 256-byte aligned
    (dict(ws_bytes=1024), -3),                        # workspace too small
])
def test_prefill_host_rejects_before_launch(L, over, code):
    count = L.loza_launch_count()
    assert _call_prefill_host(L, **over) == code
    assert L.loza_launch_count() == count


def test_prefill_host_workspace_size():
    p = bss.Params(1 / math.sqrt(576))
    size = lambda *a: bss.workspace_size(bss.LOZA_OP_PREFILL_HOST, *a)
    assert size(1, 2048, 4096, 64, 1, 576, 512, p) == 0          # max_seqlen beyond the token count
    assert size(1, 4096, 4096, 64, 4, 576, 512, p) == 0          # absorbed is one kv head
    small = size(1, 300, 300, 64, 1, 576, 512, p)
    big = size(1, 32768, 32768, 64, 1, 576, 512, p)
    huge = size(1, 1 << 20, 1 << 20, 64, 1, 576, 512, p)
    # one chunk slot at least holds the short sequence's q, latent, out and lse
    assert small >= 300 * (64 * 576 * 2 + 2 * 576 * 2 + 64 * 512 * 2 + 64 * 4)
    # chunks are bounded (at most 64 own + s + l - 1 prepended blocks, three slots)
    assert small < big <= huge
    assert huge < 3 * (71 * 128) * (64 * 576 * 2 + 64 * 512 * 2 + 2 * 576 * 2 + 64 * 4) + (256 << 20)
    # a packed batch needs slots for its longest sequence only, plus a longer chunk table
    packed = size(8, 8 * 32768, 32768, 64, 1, 576, 512, p)
    assert big <= packed < big + (1 << 20)
    # the unbounded window runs as one chunk per sequence: a slot of the longest sequence
    dense = size(1, 8192, 8192, 4, 4, 64, 64, bss.Params(0.125, n_local=bss.LOZA_UNBOUNDED))
    assert dense >= 8192 * 4 * (64 * 2 * 4 + 4)
    # other block sizes: slots of whole max(b, 128)-row units plus the chunk's prefix
    row = 64 * 576 * 2 + 64 * 512 * 2 + 2 * 576 * 2 + 64 * 4
    tok = size(1, 1 << 20, 1 << 20, 64, 1, 576, 512, bss.Params(0.1, 1, 16, 1024))  # prefix 1,152 rows
    assert huge < tok < 3 * (1152 + 8192) * row + (256 << 20)
    wide = size(1, 1 << 20, 1 << 20, 64, 1, 576, 512, bss.Params(0.1, 1024, 1, 4))
    assert wide > 3 * (4 * 1024) * 64 * 576 * 2   # prefix 4,096 rows + at least one 1,024-row unit
    assert size(1, 4096, 4096, 64, 1, 576, 512, bss.Params(0.1, 96, 1, 7)) == 0


def test_prefill_host_binding_rejects_before_any_device_work(L):
    """The binding checks dtypes, ranks and contiguity, and the shape through the
    workspace query, before it allocates or launches anything (runs without a GPU)."""
    import torch
    p = bss.Params(1 / math.sqrt(192))
    q = torch.zeros((256, 4, 576), dtype=torch.bfloat16)
    lat = torch.zeros((256, 1, 576), dtype=torch.bfloat16)
    count = L.loza_launch_count()
    with pytest.raises(TypeError):
        bss.loza_ssa_prefill_host(q.float(), lat, lat[:, :, :512], p)
    with pytest.raises(TypeError):
        bss.loza_ssa_prefill_host(q[0], lat, lat[:, :, :512], p)
    with pytest.raises(ValueError):
        bss.loza_ssa_prefill_host(q.transpose(1, 2).contiguous().transpose(1, 2), lat, lat[:, :, :512], p)
    with pytest.raises(ValueError):  # a latent V must share K's rows
        bss.loza_ssa_prefill_host(q, lat, lat.reshape(128, 2, 576)[:, :1, :512], p)
    with pytest.raises(bss.LozaError) as e:  # the whole 576-wide latent as V: no such head dims
        bss.loza_ssa_prefill_host(q, lat, lat, p)
    assert e.value.status == -2
    assert L.loza_launch_count() == count


def test_backward_window_checks(L):
    """The backward takes any bounded window whose block size is a power of
    two (it sizes a workspace for b = 64 and for the token window b = 1); a
    block size that is not a power of two and the unbounded window are
    refused (LOZA_ERR_UNSUPPORTED) before anything runs."""
    vp = ctypes.c_void_p
    for params in (bss.Params(0.125, 64, 2, 14), bss.Params(0.125, 1, 16, 1024), bss.Params(0.125, 256, 1, 3)):
        assert bss.workspace_size(bss.LOZA_OP_BACKWARD, 1, 256, 256, 4, 4, 64, 64, params) > 0
    count = L.loza_launch_count()
    for params in (bss.Params(0.125, 96, 1, 7), bss.Params(0.125, 128, 1, bss.LOZA_UNBOUNDED)):
        rc = L.loza_ssa_backward(vp(1 << 20), vp(1 << 21), vp(1 << 22), vp(1 << 23), vp(1 << 24), vp(1 << 25),
                                 vp(1 << 26), 1, 256, 256, 4, 4, 64, 64, params, vp(1 << 27), vp(1 << 28),
                                 vp(1 << 29), vp(1 << 30), 1 << 30, vp(0))
        assert rc == -2
        assert bss.workspace_size(bss.LOZA_OP_BACKWARD, 1, 256, 256, 4, 4, 64, 64, params) == 0
    assert L.loza_launch_count() == count


@pytest.mark.parametrize("limit", [0, 2000001])
def test_wait_selftest_rejects_out_of_range_limits(L, limit):
    count = L.loza_launch_count()
    assert L.loza_wait_selftest(limit, ctypes.c_void_p(0)) == -1
    assert L.loza_launch_count() == count
