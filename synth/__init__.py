"""Seeded synthetic inputs for the SSA workloads.

This module only draws random numbers and rounds them to bf16; it holds none of
the attention arithmetic. Both the fp64 oracle (through the tests and the
benchmark's CPU leg) and the CUDA library consume what it produces, so the two
sides see bit-identical inputs.

Recipe (stated once here and in the design notes):
  * values ~ N(0, 1) drawn in float32, rounded to bf16 with round-to-nearest-even
    once, on the host (numpy) or on the device (torch's float32 -> bf16 cast,
    also round-to-nearest-even);
  * host generator: numpy PCG64 seeded with 1000 + workload number; draw order
    lengths -> q -> k / latent -> v -> dO;
  * device generator (for the multi-GB workloads): torch.Generator on the device,
    seeded the same way, one call per tensor in the same order.
"""
from __future__ import annotations

import math

import numpy as np

SEED_BASE = 1000


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even. Finite inputs."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bits(gen: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) values rounded to bf16, as uint16 bit patterns."""
    return bf16_bits(gen.standard_normal(size=shape, dtype=np.float32))


def loguniform_lengths(gen: np.random.Generator, n: int, lo: int, hi: int, total_cap: int):
    """n lengths round(exp(U(ln lo, ln hi))); all n redrawn from the same stream
    while their sum exceeds total_cap."""
    while True:
        u = gen.uniform(math.log(lo), math.log(hi), size=n)
        lens = np.rint(np.exp(u)).astype(np.int64)
        lens = np.clip(lens, lo, hi)
        if int(lens.sum()) <= total_cap:
            return lens


def uniform_lengths(gen: np.random.Generator, n: int, lo: int, hi: int):
    """n integer lengths uniform on [lo, hi]."""
    return gen.integers(lo, hi, size=n, endpoint=True).astype(np.int64)


def cu_seqlens(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def torch_normal_bf16(shape, seed: int, device, chunk_elems: int = 1 << 28):
    """N(0,1) bf16 tensor drawn on ``device`` by a torch.Generator seeded with
    ``seed`` (float32 draw, then torch's round-to-nearest-even cast), filled in
    chunks to bound the float32 temporary."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e].copy_(torch.randn(e - s, generator=g, device=device, dtype=torch.float32))
    return out


# The five workloads, with their shapes (sizes as the workload definitions give them).
WORKLOADS = {
    1: dict(name="tiny MHA prefill+decode", batch=1, seqlen=2048, n_heads=4, n_kv_heads=1 * 4,
            d_qk=64, d_v=64, scale=1.0 / 8.0),
    2: dict(name="MLA-absorbed SSA prefill L=32768", batch=1, seqlen=32768, n_heads=64,
            n_kv_heads=1, d_qk=576, d_v=512, scale=1.0 / math.sqrt(192.0)),
    3: dict(name="MLA-absorbed SSA decode, 64 seqs, ctx U[65536,131072]", batch=64,
            ctx_lo=65536, ctx_hi=131072, n_heads=64, n_kv_heads=1, d_qk=576, d_v=512,
            scale=1.0 / math.sqrt(192.0)),
    4: dict(name="MLA-absorbed long prefill L=262144 and 1M decode x32", batch=1,
            seqlen=262144, decode_batch=32, decode_ctx=1 << 20, n_heads=64, n_kv_heads=1,
            d_qk=576, d_v=512, scale=1.0 / math.sqrt(192.0)),
    5: dict(name="training fwd+bwd varlen, 8 seqs log-uniform [4096,262144]", batch=8,
            len_lo=4096, len_hi=262144, total_cap=1 << 20, n_heads=64, n_kv_heads=64,
            d_qk=192, d_v=128, scale=1.0 / math.sqrt(192.0)),
}


def workload_seed(number: int) -> int:
    return SEED_BASE + number
