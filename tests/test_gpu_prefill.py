"""GPU parity of the SSA prefill kernels against the fp64 oracle.

Each case draws seeded bf16 inputs (synth), runs the CUDA path through the C ABI
and compares O and LSE element by element with the oracle on the same bits:
O max-abs <= 1e-2, mean-abs <= 1e-3; LSE max-abs <= 1e-3.
"""
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


def run_case(bss, oracle_mod, seed, lens, H, Hkv, dqk, dv, scale, n_sink=1, n_local=7, latent=False,
             rows=None):
    import torch
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
    q_dev = to_dev(q)
    cu_dev = torch.from_numpy(cu).cuda()
    params = bss.Params(scale, 128, n_sink, n_local)
    out, lse = bss.loza_ssa_prefill(q_dev, k_dev, v_dev, cu_dev, max(lens), params)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.forward(q, k_bits, v_bits, cu, H, Hkv, 128, n_sink, n_local, scale, rows=rows)
    o_got = from_dev(out)
    lse_got = lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        o_got, lse_got = o_got[rows], lse_got[rows]
    return o_got, o_ref, lse_got, lse_ref


def test_tiny_mha_d64(bss, oracle_mod):
    """Workload 1: one sequence of 2048 tokens, 4 heads, head dim 64, scale 1/8."""
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, synth.workload_seed(1), [2048], 4, 4, 64, 64, 1 / 8)
    assert_close_o(o, o_ref, "cfg1 O")
    assert_close_lse(l, l_ref, "cfg1 LSE")


@pytest.mark.parametrize("lens", [[1], [127], [128], [129], [1000, 300, 1500]])
def test_mha_d64_ragged(bss, oracle_mod, lens):
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 17 + len(lens), lens, 2, 2, 64, 64, 0.125)
    assert_close_o(o, o_ref, f"lens={lens}")
    assert_close_lse(l, l_ref, f"lens={lens}")


def test_nonabsorbed_192_128_varlen(bss, oracle_mod):
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 23, [1300, 129, 2100], 4, 4, 192, 128, 1 / math.sqrt(192))
    assert_close_o(o, o_ref, "192/128")
    assert_close_lse(l, l_ref, "192/128")


def test_absorbed_576_512_varlen(bss, oracle_mod):
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 29, [1500, 77, 1153], 4, 1, 576, 512, 1 / math.sqrt(192),
                                  latent=True)
    assert_close_o(o, o_ref, "absorbed")
    assert_close_lse(l, l_ref, "absorbed")


@pytest.mark.parametrize("n_sink,n_local", [(0, -1), (2, 3), (0, 1)])
def test_other_windows(bss, oracle_mod, n_sink, n_local):
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 31, [1200, 500], 2, 2, 64, 64, 0.125, n_sink, n_local)
    assert_close_o(o, o_ref, f"s={n_sink} l={n_local}")
    assert_close_lse(l, l_ref, f"s={n_sink} l={n_local}")


@pytest.mark.parametrize("n_sink,n_local", [(0, -1), (2, 3), (1, 1), (0, 2)])
def test_nonabsorbed_192_128_windows(bss, oracle_mod, n_sink, n_local):
    """192 / 128 (two query tiles per CTA over the union of their windows)
    with the unbounded window, several sinks, a window of one block and no
    sink; odd and even tile counts, a 1-row last tile."""
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 39, [1665, 257, 900], 2, 2, 192, 128, 1 / math.sqrt(192),
                                  n_sink, n_local)
    assert_close_o(o, o_ref, f"192/128 s={n_sink} l={n_local}")
    assert_close_lse(l, l_ref, f"192/128 s={n_sink} l={n_local}")


@pytest.mark.parametrize("n_sink,n_local", [(0, -1), (2, 3)])
def test_absorbed_other_windows(bss, oracle_mod, n_sink, n_local):
    """Absorbed shapes (CTA-pair kernel: even head count) with the unbounded and a (2, 3) window."""
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 37, [1100, 300], 2, 1, 576, 512, 1 / math.sqrt(192),
                                  n_sink, n_local, latent=True)
    assert_close_o(o, o_ref, f"absorbed s={n_sink} l={n_local}")
    assert_close_lse(l, l_ref, f"absorbed s={n_sink} l={n_local}")


def test_absorbed_odd_heads(bss, oracle_mod):
    """An odd head count runs the absorbed shapes on single CTAs."""
    o, o_ref, l, l_ref = run_case(bss, oracle_mod, 41, [700, 129], 3, 1, 576, 512, 1 / math.sqrt(192),
                                  latent=True)
    assert_close_o(o, o_ref, "absorbed, 3 heads")
    assert_close_lse(l, l_ref, "absorbed, 3 heads")


def test_absorbed_without_workspace(bss, oracle_mod):
    """Absorbed shapes with no prefill workspace: the kernel recomputes S for
    each half of the value dimension instead of keeping P between them."""
    import torch
    g = synth.rng(43)
    lens = [900, 260]
    T, H = sum(lens), 4
    cu = synth.cu_seqlens(lens)
    q = synth.normal_bits(g, (T, H, 576))
    kv = synth.normal_bits(g, (T, 1, 576))
    k_dev = to_dev(kv)
    scale = 1 / math.sqrt(192)
    out, lse = bss.loza_ssa_prefill(to_dev(q), k_dev, k_dev[:, :, :512], torch.from_numpy(cu).cuda(), max(lens),
                                    bss.Params(scale), workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.forward(q, kv, np.ascontiguousarray(kv[:, :, :512]), cu, H, 1, 128, 1, 7, scale)
    assert_close_o(from_dev(out), o_ref, "absorbed, no workspace")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "absorbed, no workspace")


@pytest.mark.parametrize("seed", [47, 53])
def test_absorbed_rescales(bss, oracle_mod, seed):
    """Absorbed shapes where the running row maximum jumps by far more than
    the lazy-rescale threshold at scattered key blocks: the 64 rotary columns
    of each key block carry a factor from {0.5, 1, 4, 8} and each head's
    queries another, so the two heads of a CTA pair rescale at different
    blocks (the quietest head rarely). The 512 value columns are halved, so
    that O stays where bf16 output rounding is below the O tolerance. Pass 2
    of the two-pass kernel must repeat exactly pass 1's rescales."""
    import torch
    g = synth.rng(seed)
    lens = [1500, 700]
    T, H = sum(lens), 4
    cu = synth.cu_seqlens(lens)
    q = synth.bits_to_f32(synth.normal_bits(g, (T, H, 576)))
    kv = synth.bits_to_f32(synth.normal_bits(g, (T, 1, 576)))
    q *= np.array([0.2, 1.0, 1.5, 0.7], np.float32)[None, :, None]
    block_f = g.choice(np.array([0.5, 1.0, 4.0, 8.0], np.float32), size=(T + 127) // 128)
    kv[:, :, 512:] *= np.repeat(block_f, 128)[:T, None, None]
    kv[:, :, :512] *= np.float32(0.5)
    q_bits, kv_bits = synth.bf16_bits(q), synth.bf16_bits(kv)
    k_dev = to_dev(kv_bits)
    scale = 1 / math.sqrt(192)
    out, lse = bss.loza_ssa_prefill(to_dev(q_bits), k_dev, k_dev[:, :, :512], torch.from_numpy(cu).cuda(),
                                    max(lens), bss.Params(scale))
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    o_ref, lse_ref = oracle_mod.forward(q_bits, kv_bits, np.ascontiguousarray(kv_bits[:, :, :512]), cu, H, 1, 128,
                                        1, 7, scale)
    assert_close_o(from_dev(out), o_ref, f"absorbed rescales seed={seed}")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, f"absorbed rescales seed={seed}")
