"""GPU parity of loza_ssa_prefill_host: the prefill of one sequence whose
tensors live in host memory, streamed through the GPU in chunks of query
blocks. Each case checks O and LSE against the fp64 oracle (same tolerances as
the device prefill) and against a device-resident loza_ssa_prefill of the same
sequence, which must agree bit for bit: every own row of a chunk is computed
by the same kernel over the same keys in the same order."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def host_bf16(bits, pinned):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


def check_host_call(bss, oracle_mod, params, qh, kh, vh, qd, kd, vd, q_bits, k_bits, v_bits, Hkv, rows=None,
                    lens=None, poison=False):
    """Run the host entry point, then compare it bit for bit with the device call
    and element by element with the oracle (on ``rows``, all rows if None).
    lens: the packed sequence lengths (one sequence of all rows if None).
    poison: hand the call a workspace of 0xFF bytes (bf16 NaN), so that any
    slot row the chunks read without writing it first shows in the outputs."""
    import torch
    L, H = qh.shape[0], qh.shape[1]
    lens = [L] if lens is None else lens
    cu_np = synth.cu_seqlens(lens)
    ws = None
    if poison:
        size = bss.workspace_size(bss.LOZA_OP_PREFILL_HOST, len(lens), L, max(lens), H, Hkv, qh.shape[2],
                                  vh.shape[2], params)
        assert size > 0
        ws = torch.full((size,), 255, dtype=torch.uint8, device="cuda")
    out_h, lse_h = bss.loza_ssa_prefill_host(qh, kh, vh, params, cu_seqlens=None if len(lens) == 1 else cu_np,
                                             workspace=ws)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    assert out_h.device.type == "cpu" and lse_h.device.type == "cpu"
    cu = torch.from_numpy(cu_np).cuda()
    out_d, lse_d = bss.loza_ssa_prefill(qd, kd, vd, cu, max(lens), params)
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16)), "O differs from the device call"
    assert torch.equal(lse_h.view(torch.int32), lse_d.cpu().view(torch.int32)), "LSE differs from the device call"
    o_ref, lse_ref = oracle_mod.forward(q_bits, k_bits, v_bits, cu_np, H, Hkv, params.block_size, params.n_sink,
                                        params.n_local, params.scale, rows=rows)
    o_got = out_h.to(torch.float32).numpy().astype(np.float64)
    lse_got = lse_h.numpy().astype(np.float64)
    if rows is not None:
        o_got, lse_got = o_got[rows], lse_got[rows]
    what = f"host L={L} d_v={vh.shape[2]}"
    assert_close_o(o_got, o_ref, what)
    assert_close_lse(lse_got, lse_ref, what)


def host_case(bss, oracle_mod, seed, L, H, Hkv, dqk, dv, scale, n_sink=1, n_local=7, latent=False,
              pinned=True, lens=None, block=128, poison=False):
    """L tokens, one sequence or packed as `lens` (summing to L)."""
    g = synth.rng(seed)
    q = synth.normal_bits(g, (L, H, dqk))
    if latent:
        kv = synth.normal_bits(g, (L, 1, dqk))
        k_bits, v_bits = kv, np.ascontiguousarray(kv[:, :, :dv])
        kh = host_bf16(kv, pinned)
        vh = kh[:, :, :dv]
        kd = to_dev(kv)
        vd = kd[:, :, :dv]
    else:
        k_bits = synth.normal_bits(g, (L, Hkv, dqk))
        v_bits = synth.normal_bits(g, (L, Hkv, dv))
        kh, vh = host_bf16(k_bits, pinned), host_bf16(v_bits, pinned)
        kd, vd = to_dev(k_bits), to_dev(v_bits)
    params = bss.Params(scale, block, n_sink, n_local)
    check_host_call(bss, oracle_mod, params, host_bf16(q, pinned), kh, vh, to_dev(q), kd, vd, q, k_bits, v_bits,
                    Hkv, lens=lens, poison=poison)


@pytest.mark.parametrize("L", [1, 200, 3000, 5000])
def test_host_absorbed(bss, oracle_mod, L):
    """Absorbed MLA (576/512 latent, v == k): 1 to 5 chunks of 8 blocks, the
    later ones with 7 prepended blocks, a ragged last block."""
    host_case(bss, oracle_mod, 400 + L, L, 4, 1, 576, 512, 1 / math.sqrt(192), latent=True)


@pytest.mark.parametrize("n_sink,n_local", [(2, 3), (0, 1), (3, 12), (0, -1)])
def test_host_windows_d64(bss, oracle_mod, n_sink, n_local):
    """Other windows: short (chunks of 8 blocks, 4 or 0 prepended), wide
    (chunks of 14 blocks), unbounded (one chunk)."""
    host_case(bss, oracle_mod, 410, 4500, 2, 2, 64, 64, 0.125, n_sink, n_local)


def test_host_192_128(bss, oracle_mod):
    host_case(bss, oracle_mod, 420, 4200, 4, 4, 192, 128, 1 / math.sqrt(192))


@pytest.mark.parametrize("lens", [[3000, 1, 700, 5000], [129, 1024, 1025, 2049, 64]])
def test_host_absorbed_packed(bss, oracle_mod, lens):
    """A packed batch: each sequence chunked on its own (1 to 5 chunks), the
    chunks of all sequences streamed through the same three slots."""
    host_case(bss, oracle_mod, 450 + len(lens), sum(lens), 4, 1, 576, 512, 1 / math.sqrt(192), latent=True,
              lens=lens)


@pytest.mark.parametrize("n_sink,n_local", [(1, 7), (2, 3), (0, -1)])
def test_host_packed_d64_and_192(bss, oracle_mod, n_sink, n_local):
    host_case(bss, oracle_mod, 460, 4300, 2, 2, 64, 64, 0.125, n_sink, n_local, lens=[2500, 300, 1500])
    host_case(bss, oracle_mod, 461, 3100, 2, 2, 192, 128, 1 / math.sqrt(192), n_sink, n_local, lens=[1100, 2000])


# (b, s, l): page 4's token window, and block sizes below and above 128; most
# leave a gap of zero rows between the sinks and the halo of a chunk's prefix
GENERAL = [(1, 16, 1024), (64, 2, 14), (256, 1, 3), (32, 3, 20), (1, 0, 300), (512, 1, 2)]


@pytest.mark.parametrize("block,n_sink,n_local", GENERAL)
def test_host_general_windows(bss, oracle_mod, block, n_sink, n_local):
    """Other block sizes: chunks of whole max(b, 128)-row units, the later ones
    on [sinks | zero gap | halo | own]; the workspace starts as NaN bytes.
    Bit for bit the device call, and the oracle."""
    host_case(bss, oracle_mod, 470 + block + n_sink, 9000, 2, 2, 64, 64, 0.125, n_sink, n_local, block=block,
              poison=True)


@pytest.mark.parametrize("block,n_sink,n_local", [(1, 16, 1024), (64, 2, 14)])
def test_host_general_windows_absorbed_and_192(bss, oracle_mod, block, n_sink, n_local):
    """The absorbed two-pass kernel and the per-head 192/128 kernel under other
    block sizes, packed batches, poisoned workspace."""
    host_case(bss, oracle_mod, 480 + block, 5600, 4, 1, 576, 512, 1 / math.sqrt(192), n_sink, n_local,
              latent=True, lens=[4000, 1, 1599], block=block, poison=True)
    host_case(bss, oracle_mod, 490 + block, 4300, 2, 2, 192, 128, 1 / math.sqrt(192), n_sink, n_local,
              lens=[2500, 300, 1500], block=block, poison=True)


def test_host_pageable(bss, oracle_mod):
    """Pageable host tensors: the copies serialise, the results are the same."""
    host_case(bss, oracle_mod, 430, 2500, 2, 2, 64, 64, 0.125, pinned=False)


def test_host_absorbed_long_64_heads(bss, oracle_mod):
    """32,768 tokens, 64 heads, absorbed: 16 chunks of 16 blocks, three slots
    in flight; bit-exact against the device call, oracle on sampled rows
    (the first, each side of some chunk boundaries, the last)."""
    import torch
    L, H, D, DV = 32768, 64, 576, 512
    qd = synth.torch_normal_bf16((L, H, D), 440, "cuda")
    latd = synth.torch_normal_bf16((L, 1, D), 441, "cuda")
    qh = torch.empty(qd.shape, dtype=torch.bfloat16, pin_memory=True)
    lath = torch.empty(latd.shape, dtype=torch.bfloat16, pin_memory=True)
    qh.copy_(qd)
    lath.copy_(latd)
    rows = np.array(sorted({0, 1, 127, 2047, 2048, 2049, 4095, 4096, 16383, 16384, 30719, 30720, L - 1}))
    lat_bits = lath.view(torch.int16).numpy().view(np.uint16)
    params = bss.Params(1 / math.sqrt(192), 128, 1, 7)
    q_bits = qh.view(torch.int16).numpy().view(np.uint16)
    check_host_call(bss, oracle_mod, params, qh, lath, lath[:, :, :DV], qd, latd, latd[:, :, :DV], q_bits, lat_bits,
                    np.ascontiguousarray(lat_bits[:, :, :DV]), 1, rows=rows)
