"""The bounded waits on the GPU: a wait that nothing completes gives up after
its limit, the host reads LOZA_ERR_TIMEOUT from the device status, and the
context stays usable (a decode right after matches the oracle)."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, from_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def test_wait_gives_up_and_reports(bss, oracle_mod):
    import time
    import torch
    assert bss.device_status() == 0
    t0 = time.perf_counter()
    assert bss.wait_selftest(20000) == -5          # 20 ms bound, nothing arrives: timed out, reported
    assert time.perf_counter() - t0 >= 0.02
    assert bss.device_status() == 0                # the read clears it
    # the context still works: an absorbed decode against the oracle
    g = synth.rng(990)
    lens = [300, 2000]
    q = synth.normal_bits(g, (2, 64, 576))
    kv = synth.normal_bits(g, (2, 2048, 1, 576))
    scale = 1.0 / math.sqrt(192.0)
    out, lse = bss.loza_ssa_decode(to_dev(q), to_dev(kv), None, torch.tensor(lens, dtype=torch.int32).cuda(), 2048,
                                   bss.Params(scale))
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.decode(q, kv, None, np.array(lens, np.int32), 64, 1, 128, 1, 7, scale, d_v=512)
    assert_close_o(from_dev(out), o_ref, "decode after a timed-out wait O")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "decode after a timed-out wait LSE")
