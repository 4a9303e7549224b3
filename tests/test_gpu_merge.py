"""GPU parity of the branch combination (LSE merge of two attention branches,
alpha-mix) against the fp64 oracle on the same bits: O max-abs <= 1e-2,
mean-abs <= 1e-3; LSE max-abs <= 1e-3; rows without keys exactly -inf."""
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


def _quarter(bits):
    """bf16 values scaled by 1/4 (exact): branch outputs of attention-like
    size, where bf16 output rounding stays below the O tolerance."""
    return synth.bf16_bits(synth.bits_to_f32(bits) * np.float32(0.25))


def _branches(seed, rows, d_v):
    g = synth.rng(seed)
    o_a = _quarter(synth.normal_bits(g, (rows, d_v)))
    o_b = _quarter(synth.normal_bits(g, (rows, d_v)))
    l_a = (g.random(rows) * 25.0 - 5.0).astype(np.float32)
    l_b = (g.random(rows) * 25.0 - 5.0).astype(np.float32)
    l_b[::11] = -np.inf          # branch b without keys
    l_a[5::13] = -np.inf         # branch a without keys
    l_a[7::97] = l_b[7::97] = -np.inf  # neither
    l_b[3::17] = l_a[3::17]      # equal weights
    return o_a, l_a, o_b, l_b


@pytest.mark.parametrize("rows,d_v", [(1, 8), (3001, 512), (777, 128)])
def test_merge_matches_oracle(bss, oracle_mod, rows, d_v):
    import torch
    o_a, l_a, o_b, l_b = _branches(100 + d_v, rows, d_v)
    out, lse = bss.loza_ssa_merge(to_dev(o_a), torch.from_numpy(l_a).cuda(), to_dev(o_b),
                                  torch.from_numpy(l_b).cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.merge(o_a, l_a.astype(np.float64), o_b, l_b.astype(np.float64))
    lse_got = lse.cpu().numpy().astype(np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_got), empty)
    assert_close_o(from_dev(out), o_ref, f"merge rows={rows} d_v={d_v}")
    assert_close_lse(lse_got[~empty], lse_ref[~empty], f"merge rows={rows} d_v={d_v}")


def test_merge_full_size_sampled(bss, oracle_mod):
    """The benchmark's shape: 32,768 tokens x 64 heads of 512 values, with the
    launch configuration the bench times; 4,096 sampled rows checked."""
    import torch
    rows, d_v = 32768 * 64, 512
    o_a = synth.torch_normal_bf16((rows, d_v), 7001, "cuda") * 0.25  # exact in bf16
    o_b = synth.torch_normal_bf16((rows, d_v), 7002, "cuda") * 0.25
    g = torch.Generator(device="cuda").manual_seed(7003)
    l_a = torch.rand(rows, device="cuda", generator=g) * 25 - 5
    l_b = torch.rand(rows, device="cuda", generator=g) * 25 - 5
    out, lse = bss.loza_ssa_merge(o_a, l_a, o_b, l_b)
    torch.cuda.synchronize()
    idx = torch.from_numpy(synth.rng(7004).choice(rows, 4096, replace=False)).cuda()
    bits = lambda t: t[idx].view(torch.int16).cpu().numpy().view(np.uint16)
    o_ref, lse_ref = oracle_mod.merge(bits(o_a), l_a[idx].double().cpu().numpy(), bits(o_b),
                                      l_b[idx].double().cpu().numpy())
    assert_close_o(from_dev(out[idx]), o_ref, "merge full size")
    assert_close_lse(lse[idx].double().cpu().numpy(), lse_ref, "merge full size")


@pytest.mark.parametrize("alpha", [0.0, 1.0, 0.3, 0.75])
def test_mix_matches_oracle(bss, oracle_mod, alpha):
    import torch
    g = synth.rng(200)
    x = _quarter(synth.normal_bits(g, (513, 64)))
    y = _quarter(synth.normal_bits(g, (513, 64)))
    out = bss.loza_ssa_mix(to_dev(x), to_dev(y), alpha)
    torch.cuda.synchronize()
    got = from_dev(out)
    assert_close_o(got, oracle_mod.mix(x, y, alpha), f"mix alpha={alpha}")
    if alpha in (0.0, 1.0):  # an input comes back bit for bit
        src = x if alpha == 1.0 else y
        assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), src)
