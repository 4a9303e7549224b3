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
    (dict(params=bss.Params(0.1, block_size=64)), -2),    # only b = 128
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
