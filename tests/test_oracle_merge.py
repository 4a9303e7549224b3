"""Pins of the oracle's branch combination (merge of two (O, LSE) branches
over disjoint key sets; alpha-mix of a full and a sparse branch) against what
the definitions fix: attention over the union of two key sets computed
directly as a softmax, empty branches, symmetry, and the mix's identities."""
import numpy as np
import pytest

import oracle
import synth


def _attn(scores, v):
    """Textbook softmax attention of one query: O, LSE (natural log)."""
    m = scores.max()
    w = np.exp(scores - m)
    return (w[:, None] * v).sum(0) / w.sum(), m + np.log(w.sum())


def _case(seed, rows=48, keys=70, d_v=40):
    g = synth.rng(seed)
    v_bits = synth.normal_bits(g, (keys, d_v))
    v = synth.bits_to_f32(v_bits).astype(np.float64)
    s = g.standard_normal((rows, keys)) * 3.0
    in_a = g.random((rows, keys)) < 0.5
    in_a[:, 0] = True  # every row keeps a key in branch a
    o_a, o_b = np.zeros((rows, d_v)), np.zeros((rows, d_v))
    l_a, l_b = np.full(rows, -np.inf), np.full(rows, -np.inf)
    o_u = np.zeros((rows, d_v))
    for r in range(rows):
        if r % 7 == 3:
            in_a[r, :] = True  # branch b empty
        a, b = in_a[r], ~in_a[r]
        o_a[r], l_a[r] = _attn(s[r, a], v[a])
        if b.any():
            o_b[r], l_b[r] = _attn(s[r, b], v[b])
        o_u[r], _ = _attn(s[r], v)
    return o_a, l_a, o_b, l_b, o_u, s, v


def test_merge_equals_attention_over_the_union():
    o_a, l_a, o_b, l_b, o_u, s, v = _case(1)
    # the branch outputs enter as bf16, as a kernel would write them
    oa_bits, ob_bits = synth.bf16_bits(o_a.astype(np.float32)), synth.bf16_bits(o_b.astype(np.float32))
    o, lse = oracle.merge(oa_bits, l_a, ob_bits, l_b)
    lse_u = np.array([sr.max() + np.log(np.exp(sr - sr.max()).sum()) for sr in s])
    np.testing.assert_allclose(lse, lse_u, rtol=0, atol=1e-12)
    # the only difference left is the bf16 rounding of the branch outputs (|O| <= max|v|)
    assert np.abs(o - o_u).max() <= 2.0 ** -8 * np.abs(v).max()


def test_merge_with_an_empty_branch_is_the_other_branch():
    o_a, l_a, o_b, l_b, _, _, _ = _case(2)
    oa_bits = synth.bf16_bits(o_a.astype(np.float32))
    ob_bits = synth.bf16_bits(o_b.astype(np.float32))
    empty = np.full_like(l_b, -np.inf)
    o, lse = oracle.merge(oa_bits, l_a, ob_bits, empty)
    np.testing.assert_array_equal(lse, l_a)
    np.testing.assert_array_equal(o, synth.bits_to_f32(oa_bits).astype(np.float64))


def test_merge_of_two_empty_branches():
    bits = synth.normal_bits(synth.rng(3), (4, 8))
    inf = np.full(4, -np.inf)
    o, lse = oracle.merge(bits, inf, bits, inf)
    assert np.all(lse == -np.inf) and np.all(o == 0.0)


def test_merge_is_symmetric():
    o_a, l_a, o_b, l_b, _, _, _ = _case(4)
    oa_bits = synth.bf16_bits(o_a.astype(np.float32))
    ob_bits = synth.bf16_bits(o_b.astype(np.float32))
    o1, l1 = oracle.merge(oa_bits, l_a, ob_bits, l_b)
    o2, l2 = oracle.merge(ob_bits, l_b, oa_bits, l_a)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-15)


@pytest.mark.parametrize("alpha", [0.0, 1.0, 0.3])
def test_mix_identities(alpha):
    g = synth.rng(5)
    x = synth.normal_bits(g, (6, 16))
    y = synth.normal_bits(g, (6, 16))
    xf = synth.bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(oracle.mix(x, x, alpha), xf, rtol=0, atol=1e-15)  # a x + (1-a) x = x
    if alpha == 1.0:
        np.testing.assert_array_equal(oracle.mix(x, y, alpha), xf)
    if alpha == 0.0:
        np.testing.assert_array_equal(oracle.mix(x, y, alpha), synth.bits_to_f32(y).astype(np.float64))
