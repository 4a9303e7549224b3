"""Pins of the fp64 oracle against what the definition and mathematics fix.

None of these compares the oracle with itself under a retyped formula: each
check uses an independent route (a library routine with an explicit mask, a
brute-force enumeration written from the token-distance form of the window, a
closed form, or an invariant of softmax attention). The definition is the one
stated by Efficient Context Scaling with LongCat ZigZag Attention, page 1
section 01 (sink + local blocks, b = 128, s = 1, l = 7), page 2 section 2.2 and
page 5 (1 + 7 blocks of 128 tokens = 1,024-token window).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(bits):
    return synth.bits_to_f32(bits).astype(np.float64)


def allowed_mask(L, b, s, l):
    """Token-distance form of the window: key t visible from query i iff
    t <= i and (t's block is a sink block, or the block distance is < l)."""
    i = np.arange(L)[:, None]
    t = np.arange(L)[None, :]
    local = (i // b - t // b) < l if l >= 0 else np.ones((L, L), bool)
    return (t <= i) & ((t // b < s) | local)


def packed_mask(lens, b, s, l):
    T = int(sum(lens))
    m = np.zeros((T, T), bool)
    o = 0
    for L in lens:
        m[o:o + L, o:o + L] = allowed_mask(L, b, s, l)
        o += L
    return m


def sdpa_ref(q, k, v, mask, scale):
    """torch fp64 scaled_dot_product_attention with an explicit boolean mask.
    q [T,H,d], k/v [T,Hkv,d]. Returns O [T,H,dv], LSE [T,H]."""
    H, Hkv = q.shape[1], k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)[None]
    mt = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt, scale=scale)
    logits = torch.einsum("bhid,bhtd->bhit", qt, kt) * scale
    lse = torch.logsumexp(logits.masked_fill(~mt, float("-inf")), dim=-1)
    return o[0].permute(1, 0, 2).numpy(), lse[0].permute(1, 0).numpy()


def make_problem(seed, lens, H, Hkv, dqk, dv):
    g = synth.rng(seed)
    T = int(sum(lens))
    q = synth.normal_bits(g, (T, H, dqk))
    k = synth.normal_bits(g, (T, Hkv, dqk))
    v = synth.normal_bits(g, (T, Hkv, dv))
    return q, k, v, synth.cu_seqlens(lens)


# ---- p3: brute force on tiny shapes ---------------------------------------

@pytest.mark.parametrize("s,l", [(1, 2), (2, 3), (0, 1), (1, 7), (3, 1)])
@pytest.mark.parametrize("Hkv", [1, 2])
def test_bruteforce_tiny(oracle_mod, s, l, Hkv):
    b, H, dqk, dv = 4, 2, 8, 6
    lens = [37, 64, 5]                      # ragged tails, blocks restart per sequence
    q, k, v, cu = make_problem(7 + s * 10 + l, lens, H, Hkv, dqk, dv)
    scale = 0.3
    o, lse = oracle_mod.forward(q, k, v, cu, H, Hkv, b, s, l, scale)
    qf, kf, vf = f64(q), f64(k), f64(v)
    for n, L in enumerate(lens):
        base = cu[n]
        for i in range(L):
            for h in range(H):
                hk = h // (H // Hkv)
                num = np.zeros(dv)
                den = 0.0
                for t in range(L):
                    if not (t <= i and (t // b < s or i // b - t // b < l)):
                        continue
                    w = math.exp(scale * float(qf[base + i, h] @ kf[base + t, hk]))
                    num += w * vf[base + t, hk]
                    den += w
                np.testing.assert_allclose(o[base + i, h], num / den, rtol=1e-12, atol=1e-12)
                assert abs(lse[base + i, h] - math.log(den)) < 1e-12


# ---- p2 / p6: explicit-mask library attention -----------------------------

@pytest.mark.parametrize("b,s,l,lens", [
    (128, 1, 7, [2048]),
    (16, 1, 3, [300, 129, 17]),
    (16, 2, 2, [200]),
    (32, 0, 1, [150, 70]),           # block-diagonal causal
    (32, 0, -1, [150, 70]),          # unbounded: plain causal
])
def test_matches_masked_sdpa(oracle_mod, b, s, l, lens):
    H, Hkv, dqk, dv = 4, 1 if s != 2 else 4, 32, 24
    q, k, v, cu = make_problem(11 + b + s + l, lens, H, Hkv, dqk, dv)
    scale = 1.0 / math.sqrt(dqk)
    o, lse = oracle_mod.forward(q, k, v, cu, H, Hkv, b, s, l, scale)
    o_ref, lse_ref = sdpa_ref(f64(q), f64(k), f64(v), packed_mask(lens, b, s, l), scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-11)


def test_unbounded_window_is_torch_causal(oracle_mod):
    L, H, d = 333, 3, 16
    q, k, v, cu = make_problem(5, [L], H, H, d, d)
    o, _ = oracle_mod.forward(q, k, v, cu, H, H, 16, 0, -1, 0.25)
    qt = torch.from_numpy(f64(q)).permute(1, 0, 2)[None]
    kt = torch.from_numpy(f64(k)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(f64(v)).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.25)
    np.testing.assert_allclose(o, ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-11)


# ---- p1: up to (s+l)*b tokens SSA is full causal attention ----------------

def test_short_sequences_are_full_causal(oracle_mod):
    b, s, l = 128, 1, 7
    H, d = 2, 16
    lens = [1024, 700, 1]
    q, k, v, cu = make_problem(3, lens, H, H, d, d)
    o, lse = oracle_mod.forward(q, k, v, cu, H, H, b, s, l, 0.2)
    # plain causal softmax attention written directly (no blocks anywhere)
    qf, kf, vf = f64(q), f64(k), f64(v)
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        for h in range(H):
            z = 0.2 * qf[sl, h] @ kf[sl, h].T
            z[np.triu_indices(L, 1)] = -np.inf
            m = z.max(axis=1, keepdims=True)
            w = np.exp(z - m)
            np.testing.assert_allclose(o[sl, h], (w @ vf[sl, h]) / w.sum(1, keepdims=True),
                                       rtol=0, atol=1e-11)
            np.testing.assert_allclose(lse[sl, h], m[:, 0] + np.log(w.sum(1)), rtol=0, atol=1e-11)


# ---- p4: window counts ------------------------------------------------------

def closed_form_count(i, b=128, s=1, l=7):
    return i + 1 if i // b < s + l - 1 else s * b + (l - 1) * b + (i % b) + 1


def test_window_counts_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "window_counts.json")))
    b, s, l = g["block_size"], g["n_sink"], g["n_local"]
    for L, total in g["pairs_per_sequence"].items():
        L = int(L)
        # closed form summed block by block
        acc = 0
        for j in range((L + b - 1) // b):
            lo, hi = j * b, min(L, (j + 1) * b)
            if j < s + l - 1:
                acc += sum(i + 1 for i in range(lo, hi))
            else:
                acc += (hi - lo) * (s * b + (l - 1) * b + 1) + sum(i % b for i in range(lo, hi))
        assert acc == total
    rs = np.random.default_rng(0)
    for i in list(range(0, 1200, 7)) + list(rs.integers(0, 1 << 20, 200)):
        c = oracle_mod.visible_count(int(i), b, s, l)
        assert c == closed_form_count(int(i), b, s, l)
        assert c <= g["max_keys_per_query"]


def test_zero_query_gives_uniform_weights(oracle_mod):
    """q = 0: every visible key gets the same weight, so O is the mean of v over
    A(i) and LSE = ln |A(i)|; summing exp(LSE) over a sequence gives the pair count."""
    b, s, l = 128, 1, 7
    L, H, d = 2048, 1, 8
    g = synth.rng(9)
    q = np.zeros((L, H, d), np.uint16)
    k = synth.normal_bits(g, (L, 1, d))
    v = synth.normal_bits(g, (L, 1, d))
    cu = synth.cu_seqlens([L])
    o, lse = oracle_mod.forward(q, k, v, cu, H, 1, b, s, l, 1.0)
    counts = np.exp(lse[:, 0])
    assert abs(counts.sum() - 1508352) < 1e-6
    vf = f64(v)[:, 0]
    for i in [0, 5, 127, 128, 900, 1023, 1024, 1100, 2047]:
        vis = [t for t in range(i + 1) if t // b < s or i // b - t // b < l]
        np.testing.assert_allclose(o[i, 0], vf[vis].mean(0), rtol=0, atol=1e-12)
        assert abs(counts[i] - len(vis)) < 1e-9


def test_constant_values_and_logit_shift(oracle_mod):
    b, s, l = 8, 1, 2
    L, H, d = 50, 2, 4
    g = synth.rng(4)
    # small multiples of 1/8 are exact in bf16, so k + u stays exact
    qv = (g.integers(-4, 5, (L, H, d)) / 8).astype(np.float32)
    kv = (g.integers(-4, 5, (L, 1, d)) / 8).astype(np.float32)
    u = (g.integers(-4, 5, (1, 1, d)) / 8).astype(np.float32)
    q, k, k2 = synth.bf16_bits(qv), synth.bf16_bits(kv), synth.bf16_bits(kv + u)
    cu = synth.cu_seqlens([L])
    c = np.full((L, 1, d), 1.5, np.float32)
    o, _ = oracle_mod.forward(q, k, synth.bf16_bits(c), cu, H, 1, b, s, l, 0.7)
    np.testing.assert_allclose(o, 1.5, rtol=0, atol=1e-12)
    v = synth.normal_bits(g, (L, 1, d))
    o1, lse1 = oracle_mod.forward(q, k, v, cu, H, 1, b, s, l, 0.7)
    o2, lse2 = oracle_mod.forward(q, k2, v, cu, H, 1, b, s, l, 0.7)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    shift = 0.7 * (f64(q) @ f64(synth.bf16_bits(u))[0, 0])
    np.testing.assert_allclose(lse2 - lse1, shift, rtol=0, atol=1e-12)


def test_packed_sequences_are_independent(oracle_mod):
    lens = [300, 129, 517]
    H, d = 2, 16
    q, k, v, cu = make_problem(21, lens, H, 1, d, d)
    o, lse = oracle_mod.forward(q, k, v, cu, H, 1, 32, 1, 3, 0.25)
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        o1, lse1 = oracle_mod.forward(q[sl], k[sl], v[sl], synth.cu_seqlens([L]), H, 1, 32, 1, 3, 0.25)
        np.testing.assert_array_equal(o[sl], o1)
        np.testing.assert_array_equal(lse[sl], lse1)


def test_row_subset_matches_full(oracle_mod):
    q, k, v, cu = make_problem(2, [400, 77], 2, 1, 16, 8)
    o, lse = oracle_mod.forward(q, k, v, cu, 2, 1, 16, 1, 3, 0.3)
    rows = np.array([0, 5, 399, 400, 476, 200])
    o2, lse2 = oracle_mod.forward(q, k, v, cu, 2, 1, 16, 1, 3, 0.3, rows=rows)
    np.testing.assert_array_equal(o[rows], o2)
    np.testing.assert_array_equal(lse[rows], lse2)


# ---- p7: decode is the last row of prefill ---------------------------------

@pytest.mark.parametrize("lens", [[2048], [1, 128, 129, 1000, 1025]])
def test_decode_is_last_prefill_row(oracle_mod, lens):
    b, s, l = 128, 1, 7
    H, Hkv, dqk, dv = 4, 1, 24, 16
    g = synth.rng(31)
    Lcap = max(lens) + 3
    B = len(lens)
    kc = synth.normal_bits(g, (B, Lcap, Hkv, dqk))
    vc = synth.normal_bits(g, (B, Lcap, Hkv, dv))
    qd = synth.normal_bits(g, (B, H, dqk))
    od, lsed = oracle_mod.decode(qd, kc, vc, np.array(lens, np.int32), H, Hkv, b, s, l, 0.2)
    for n, L in enumerate(lens):
        q = np.zeros((L, H, dqk), np.uint16)
        q[L - 1] = qd[n]
        o, lse = oracle_mod.forward(q, kc[n, :L], vc[n, :L], synth.cu_seqlens([L]), H, Hkv,
                                    b, s, l, 0.2, rows=np.array([L - 1]))
        np.testing.assert_allclose(od[n], o[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lsed[n], lse[0], rtol=0, atol=1e-13)


# ---- p8: gradients ----------------------------------------------------------

def autograd_ref(q, k, v, dout, lens, b, s, l, scale):
    """Gradients of sum(O * dO) by torch autograd through fp64 masked SDPA."""
    H, Hkv = q.shape[1], k.shape[1]
    qt = torch.from_numpy(q).requires_grad_(True)
    kt = torch.from_numpy(k).requires_grad_(True)
    vt = torch.from_numpy(v).requires_grad_(True)
    mask = torch.from_numpy(packed_mask(lens, b, s, l))
    kk = kt.repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)[None]
    vv = vt.repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt.permute(1, 0, 2)[None], kk, vv, attn_mask=mask, scale=scale)
    (o[0].permute(1, 0, 2) * torch.from_numpy(dout)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("b,s,l,lens,H,Hkv", [
    (4, 1, 2, [40], 2, 2),
    (4, 2, 3, [23, 40], 2, 1),
    (16, 1, 7, [300, 150], 3, 3),
    (8, 0, -1, [50], 2, 1),
])
def test_backward_matches_autograd(oracle_mod, b, s, l, lens, H, Hkv):
    dqk, dv = 12, 8
    q, k, v, cu = make_problem(41 + b + s, lens, H, Hkv, dqk, dv)
    g = synth.rng(99)
    dout = synth.normal_bits(g, (int(cu[-1]), H, dv))
    scale = 0.35
    dq, dk, dvv = oracle_mod.backward(q, k, v, dout, cu, H, Hkv, b, s, l, scale)
    rq, rk, rv = autograd_ref(f64(q), f64(k), f64(v), f64(dout), lens, b, s, l, scale)
    np.testing.assert_allclose(dq, rq, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, rk, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dvv, rv, rtol=0, atol=1e-11)


def test_backward_invariants(oracle_mod):
    """Rows of P sum to one, so sum_t dV_t = sum_i sum_h dO_i; adding one vector to
    every key leaves O unchanged, so sum_t dK_t = 0 per sequence and kv head;
    constant keys give dQ = 0."""
    lens = [260, 99]
    H, Hkv, dqk, dv = 4, 1, 16, 8
    q, k, v, cu = make_problem(77, lens, H, Hkv, dqk, dv)
    g = synth.rng(78)
    dout = synth.normal_bits(g, (int(cu[-1]), H, dv))
    dq, dk, dvv = oracle_mod.backward(q, k, v, dout, cu, H, Hkv, 32, 1, 3, 0.25)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        np.testing.assert_allclose(dvv[sl].sum(axis=(0, 1)), f64(dout)[sl].sum(axis=(0, 1)),
                                   rtol=0, atol=1e-10)
        np.testing.assert_allclose(dk[sl].sum(axis=(0, 1)), 0.0, rtol=0, atol=1e-10)
    kconst = np.broadcast_to(k[:1], k.shape).copy()
    dq0, _, _ = oracle_mod.backward(q, kconst, v, dout, cu, H, Hkv, 32, 1, 3, 0.25)
    np.testing.assert_allclose(dq0, 0.0, rtol=0, atol=1e-12)


def test_backward_row_subsets(oracle_mod):
    lens = [200, 70]
    q, k, v, cu = make_problem(55, lens, 2, 2, 8, 8)
    dout = synth.normal_bits(synth.rng(56), (270, 2, 8))
    dq, dk, dv = oracle_mod.backward(q, k, v, dout, cu, 2, 2, 16, 1, 2, 0.3)
    qr = np.array([0, 17, 199, 200, 269])
    kr = np.array([0, 15, 16, 150, 200, 210])
    dq2, dk2, dv2 = oracle_mod.backward(q, k, v, dout, cu, 2, 2, 16, 1, 2, 0.3,
                                        q_rows=qr, k_rows=kr)
    np.testing.assert_array_equal(dq[qr], dq2)
    np.testing.assert_allclose(dk[kr], dk2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv[kr], dv2, rtol=0, atol=1e-13)


def test_oracle_rejects_bad_arguments(oracle_mod):
    q, k, v, cu = make_problem(1, [10], 3, 2, 4, 4)
    with pytest.raises(ValueError):
        oracle_mod.forward(q, k, v, cu, 3, 2, 4, 1, 1, 1.0)       # 3 % 2 != 0
    with pytest.raises(ValueError):
        oracle_mod.forward(q, k, v, cu, 3, 3, 4, 1, 1, 1.0, rows=np.array([10]))
    with pytest.raises(TypeError):
        oracle_mod.forward(q.astype(np.float32), k, v, cu, 3, 3, 4, 1, 1, 1.0)


def test_latent_decode_reads_cache_in_place(oracle_mod):
    """A latent cache passed once (V = its first d_v columns) gives the same result
    as a separate, copied V cache."""
    g = synth.rng(91)
    B, Lcap, H, D, DV = 3, 700, 4, 24, 16
    kc = synth.normal_bits(g, (B, Lcap, 1, D))
    qd = synth.normal_bits(g, (B, H, D))
    lens = np.array([1, 300, 700], np.int32)
    o1, l1 = oracle_mod.decode(qd, kc, np.ascontiguousarray(kc[..., :DV]), lens, H, 1, 128, 1, 7, 0.3)
    o2, l2 = oracle_mod.decode(qd, kc, None, lens, H, 1, 128, 1, 7, 0.3, d_v=DV)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
