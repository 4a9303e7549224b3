"""Pins of the oracle's token-granular window (page 4, the LSA article's
streaming-aware index: every query keeps a fixed set of sink tokens and a
sliding window of recent tokens, 16 + 1,024 there):
    A(i) = { t <= i : t < sink_tokens  or  i - t < window_tokens }.
Each pin compares with something other than that formula: the block oracle
(whose key lists come from a different routine) where the two windows select
the same keys, closed forms, and the counts |A(i)|."""
import math

import numpy as np
import pytest

import synth


def draw(seed, T, H, Hkv, dqk, dv):
    g = synth.rng(seed)
    return (synth.normal_bits(g, (T, H, dqk)), synth.normal_bits(g, (T, Hkv, dqk)),
            synth.normal_bits(g, (T, Hkv, dv)))


def token_count(i, sink, window):
    """|A(i)|: the window's min(i + 1, W) most recent tokens plus the sink
    tokens that lie before the window."""
    in_window = min(i + 1, window)
    return in_window + max(0, min(sink, i + 1 - window))


def test_block_ends_equal_the_block_window(oracle_mod):
    """At the last row of a block (i = 128j + 127) the 1,024 most recent tokens
    are exactly blocks j-7 .. j, and 128 sink tokens are block 0: the token
    window equals the block window (b, s, l) = (128, 1, 8) there."""
    T, H = 2304, 2
    q, k, v = draw(501, T, H, H, 16, 16)
    cu = synth.cu_seqlens([T])
    rows = np.arange(127, T, 128)
    o_t, l_t = oracle_mod.forward_tokens(q, k, v, cu, H, H, 128, 1024, 0.25, rows=rows)
    o_b, l_b = oracle_mod.forward(q, k, v, cu, H, H, 128, 1, 8, 0.25, rows=rows)
    np.testing.assert_allclose(o_t, o_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_t, l_b, rtol=0, atol=1e-12)


def test_other_rows_differ_from_the_block_window(oracle_mod):
    """Inside a block the token window has dropped the oldest tokens of block
    j-8 .. j-7 that the block window still holds (or holds ones it lacks): the two
    must differ there, or the token window would not be token-granular."""
    T, H = 1600, 1
    q, k, v = draw(502, T, H, H, 16, 16)
    cu = synth.cu_seqlens([T])
    rows = np.array([1300, 1400, 1500])  # window starts 277, 377, 477: past the sink block, not on a block edge
    _, l_t = oracle_mod.forward_tokens(q, k, v, cu, H, H, 128, 1024, 0.25, rows=rows)
    _, l_b = oracle_mod.forward(q, k, v, cu, H, H, 128, 1, 8, 0.25, rows=rows)
    assert np.all(np.abs(l_t - l_b) > 1e-6)


@pytest.mark.parametrize("sink,window", [(0, 5000), (16, 4096), (3, 10 ** 9)])
def test_window_over_everything_is_causal_attention(oracle_mod, sink, window):
    """A window at least as long as the sequence: plain causal attention, the
    block oracle's unbounded window (packed sequences, two kv-head groups)."""
    lens = [700, 1, 129, 2000]
    T, H, Hkv = sum(lens), 4, 2
    q, k, v = draw(503, T, H, Hkv, 32, 24)
    cu = synth.cu_seqlens(lens)
    o_t, l_t = oracle_mod.forward_tokens(q, k, v, cu, H, Hkv, sink, window, 1 / math.sqrt(32))
    o_b, l_b = oracle_mod.forward(q, k, v, cu, H, Hkv, 128, 0, -1, 1 / math.sqrt(32))
    np.testing.assert_allclose(o_t, o_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_t, l_b, rtol=0, atol=1e-12)


def test_window_of_one_without_sinks_sees_itself(oracle_mod):
    """W = 1, no sinks: each query sees only its own key, so O_i = v_i exactly
    and LSE_i = scale * q_i . k_i."""
    T, H = 300, 2
    q, k, v = draw(504, T, H, H, 8, 8)
    cu = synth.cu_seqlens([T])
    o, lse = oracle_mod.forward_tokens(q, k, v, cu, H, H, 0, 1, 0.5)
    qf, kf, vf = (synth.bits_to_f32(x).astype(np.float64) for x in (q, k, v))
    np.testing.assert_array_equal(o, vf)
    np.testing.assert_allclose(lse, 0.5 * np.einsum("thd,thd->th", qf, kf), rtol=0, atol=1e-12)


@pytest.mark.parametrize("sink,window", [(16, 1024), (4, 32), (0, 7), (40, 1)])
def test_counts_through_zero_queries(oracle_mod, sink, window):
    """q = 0 makes every visible logit 0: exp(LSE_i) = |A(i)|, which has the
    closed form min(i+1, W) + max(0, min(S, i+1-W)), and O_i is the mean of v
    over A(i) (here with v = the key position, so the mean has a closed form too)."""
    T = 1500 if window > 100 else 200
    q = np.zeros((T, 1, 8), np.uint16)  # bf16 +0.0
    k = synth.normal_bits(synth.rng(505), (T, 1, 8))
    pos = np.arange(T, dtype=np.float32)
    v = synth.bf16_bits(np.repeat(pos[:, None, None], 8, axis=2))  # positions < 256 are exact in bf16
    cu = synth.cu_seqlens([T])
    o, lse = oracle_mod.forward_tokens(q, k, v, cu, 1, 1, sink, window, 1.0)
    counts = np.array([token_count(i, sink, window) for i in range(T)], np.float64)
    np.testing.assert_allclose(np.exp(lse[:, 0]), counts, rtol=1e-12)
    for i in (0, 1, sink, window - 1, window, window + sink, T - 1):
        if not 0 <= i < min(T, 256):
            continue
        keys = [t for t in range(i + 1) if t < sink or i - t < window]
        assert o[i, 0, 0] == pytest.approx(np.mean(keys), abs=1e-12)
    assert max(counts) <= sink + window


def test_rejects_bad_windows(oracle_mod):
    q, k, v = draw(506, 10, 1, 1, 8, 8)
    cu = synth.cu_seqlens([10])
    with pytest.raises(ValueError):
        oracle_mod.forward_tokens(q, k, v, cu, 1, 1, 0, 0, 1.0)
    with pytest.raises(ValueError):
        oracle_mod.forward_tokens(q, k, v, cu, 1, 1, -1, 4, 1.0)


@pytest.mark.parametrize("sink,window", [(16, 1024), (0, 300), (5, 1)])
def test_token_window_is_the_block_window_with_single_token_blocks(oracle_mod, sink, window):
    """With blocks of one token, s sink blocks and l local blocks select the
    tokens t < s and i - l < t <= i: the token window of S = s sink tokens and a
    W = l token sliding window. The block oracle (b = 1) and the token oracle
    list their keys by different routines; they must agree on every row of a
    packed batch."""
    lens = [2500, 1, 700]
    T, H = sum(lens), 2
    q, k, v = draw(510 + window, T, H, H, 16, 16)
    cu = synth.cu_seqlens(lens)
    o_t, l_t = oracle_mod.forward_tokens(q, k, v, cu, H, H, sink, window, 0.25)
    o_b, l_b = oracle_mod.forward(q, k, v, cu, H, H, 1, sink, window, 0.25)
    np.testing.assert_allclose(o_t, o_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_t, l_b, rtol=0, atol=1e-12)
