"""The decode entry point for callers that cannot allocate device memory.

loza_ssa_decode_noalloc serves callers such as a plug-in whose host
application owns the device allocator, or a serving runtime that reserved all
device memory for its own pool: it takes no workspace and keeps its split-KV
partials in a fixed array inside the library (the unbounded window is the
decode that needs such scratch; the 1 + 7 window merges on chip). These tests
call it through the C ABI and check it against loza_ssa_decode (which uses a
caller-provided workspace) on two calls in a row per window, so the second
call also shows that the shared array is correctly reused. This file is
collected last on purpose.
"""
import ctypes
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, from_dev, to_dev


def _inputs(seed, lens, Lcap):
    import torch
    g = synth.rng(seed)
    B, H, D = len(lens), 64, 576
    q = to_dev(synth.normal_bits(g, (B, H, D)))
    cache = to_dev(synth.normal_bits(g, (B, Lcap, 1, D)))
    seqlens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, cache, seqlens


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_twice():
    import torch
    import block_sparse_streaming_b200 as bss
    bss.build()
    windows = [bss.Params(1.0 / math.sqrt(192.0)),                          # 1 + 7 window
               bss.Params(1.0 / math.sqrt(192.0), 128, 0, bss.LOZA_UNBOUNDED)]  # needs the scratch array
    cases = [(71, [1, 130, 1025, 3000], 3072), (72, [3072, 7, 2000], 3072)]
    for params, (seed, lens, Lcap) in [(w, c) for w in windows for c in cases]:  # two calls in a row each
        q, cache, seqlens = _inputs(seed, lens, Lcap)
        ref_o, ref_l = bss.loza_ssa_decode(q, cache, None, seqlens, Lcap, params)
        out = torch.empty_like(ref_o)
        lse = torch.empty_like(ref_l)
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        free_before, _ = torch.cuda.mem_get_info()    # device-wide: any allocation by anyone
        bss.loza_ssa_decode_noalloc(q, cache, None, seqlens, Lcap, params, out, lse)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert torch.cuda.mem_get_info()[0] == free_before
        assert bss.device_status() == 0
        assert_close_o(from_dev(out), from_dev(ref_o), "noalloc vs workspace decode O")
        assert_close_lse(lse.cpu().numpy().astype(np.float64), ref_l.cpu().numpy().astype(np.float64),
                         "noalloc vs workspace decode LSE")
        # the same plan on the same data: the results agree bit for bit
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)


def test_noalloc_decode_rejects_batch_beyond_builtin_scratch():
    """4 sequences of up to 4,096 tokens with the unbounded window need more than
    the 16 MiB built in: rejected with LOZA_ERR_WORKSPACE before anything runs
    (no GPU needed). q is NULL: had the size check been skipped, the argument
    check would refuse the call (LOZA_ERR_INVALID_ARG) before any launch."""
    import block_sparse_streaming_b200 as bss
    bss.build()
    L = bss.lib()
    vp = ctypes.c_void_p
    count = L.loza_launch_count()
    rc = L.loza_ssa_decode_noalloc(vp(0), vp(1 << 21), vp(0), vp(1 << 22), 4, 4096, 4096 * 576, 576,
                                   64, 1, 576, 512, bss.Params(0.07, 128, 0, bss.LOZA_UNBOUNDED), vp(1 << 23),
                                   vp(1 << 24), vp(0))
    assert rc == -3
    assert L.loza_launch_count() == count
