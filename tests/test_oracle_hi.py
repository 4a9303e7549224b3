"""Pins of the oracle's hierarchical index decode (page 4, "LongCat Sparse
Attention", its hierarchical index: pages of 128 tokens scored coarsely, the
top pages recalled, then their tokens scored one by one and the best kept; its
streaming-aware index: fixed sink and window tokens plus those dynamic tokens,
the two parts merged by their log-sum-exp).

The oracle computes the index scores in fp32 exactly as the kernels do. The
pins use index keys and queries of small integers, for which every score and
page mean is exact in any precision and any order, so that numpy's own
arithmetic and sort (a library routine) give the reference selection; and
the limits where the hierarchical index must reduce to a flat one, to plain
SSA, or to full causal attention."""
import numpy as np
import pytest

import synth


def int_bits(g, shape, lo=-3, hi=3):
    """bf16 bit patterns of small integers (exact in bf16)."""
    return synth.bf16_bits(g.integers(lo, hi + 1, size=shape).astype(np.float32))


def in_window(t, i, b, s, l):
    if t > i:
        return False
    if l < 0 or t < s * b:
        return True
    return t >= max(0, (i // b - l + 1) * b)


def numpy_select(q_idx, k_idx, seqlens, b, s, l, top_pages, top_k):
    """Reference selection with numpy: exact scores (small integers), stable
    sort by (score descending, index ascending)."""
    B, Lcap, d = k_idx.shape
    qf = synth.bits_to_f32(q_idx).astype(np.float64)
    kf = synth.bits_to_f32(k_idx).astype(np.float64)
    out = np.full((B, top_k), -1, np.int32)
    for n, L in enumerate(seqlens):
        i = L - 1
        full = L // 128
        cand = [p for p in range(full) if any(not in_window(p * 128 + r, i, b, s, l) for r in range(128))]
        if not cand or top_k == 0 or top_pages == 0:
            continue
        ps = np.array([qf[n] @ kf[n, p * 128:(p + 1) * 128].mean(axis=0) for p in cand])
        order = np.lexsort((np.array(cand), -ps))
        pages = [cand[o] for o in order[:top_pages]]
        toks = [p * 128 + r for p in pages for r in range(128) if not in_window(p * 128 + r, i, b, s, l)]
        ts = np.array([qf[n] @ kf[n, t] for t in toks])
        order = np.lexsort((np.array(toks), -ts))
        chosen = sorted(toks[o] for o in order[:top_k])
        out[n, :len(chosen)] = chosen
    return out


def test_page_keys_are_page_means(oracle_mod):
    g = synth.rng(801)
    k = int_bits(g, (3, 1000, 16))
    lens = [1000, 256, 127]
    pk = oracle_mod.hi_page_keys(k, lens)
    kf = synth.bits_to_f32(k).astype(np.float64)
    for n, L in enumerate(lens):
        for p in range(L // 128):
            np.testing.assert_array_equal(pk[n, p], kf[n, p * 128:(p + 1) * 128].mean(axis=0))
    assert not pk[2].any()  # a sequence shorter than a page has no whole page


@pytest.mark.parametrize("win,top_pages,top_k", [((1, 16, 1024), 3, 200), ((128, 1, 2), 5, 64),
                                                  ((64, 2, 3), 100, 1000), ((1, 0, 50), 2, 7)])
def test_select_matches_numpy_on_exact_scores(oracle_mod, win, top_pages, top_k):
    """Small-integer keys and queries: every score is exact, so the oracle's
    fp32 selection must equal numpy's, ties to the lower index included (there
    are many ties: scores are small integers)."""
    b, s, l = win
    g = synth.rng(802 + top_k)
    B, Lcap, d = 3, 3000, 16
    q = int_bits(g, (B, d))
    k = int_bits(g, (B, Lcap, d))
    lens = [3000, 1500, 900]
    pk = oracle_mod.hi_page_keys(k, lens)
    got = oracle_mod.hi_select(q, k, pk, lens, b, s, l, top_pages, top_k)
    ref = numpy_select(q, k, lens, b, s, l, top_pages, top_k)
    np.testing.assert_array_equal(got, ref)


def test_all_pages_recalled_is_the_flat_index(oracle_mod):
    """With at least as many recalled pages as pages, the two stages reduce to
    one flat top-k over every token outside the window (random bf16 keys: the
    flat reference scores with the same fp32 multiply-adds, summed in order)."""
    g = synth.rng(803)
    B, Lcap, d = 2, 4096, 32
    q = synth.normal_bits(g, (B, d))
    k = synth.normal_bits(g, (B, Lcap, d))
    lens = [4096, 2300]
    pk = oracle_mod.hi_page_keys(k, lens)
    top_k = 300
    got = oracle_mod.hi_select(q, k, pk, lens, 1, 16, 1024, 10 ** 6, top_k)
    qf, kf = synth.bits_to_f32(q), synth.bits_to_f32(k)
    for n, L in enumerate(lens):
        full = (L // 128) * 128
        toks = [t for t in range(full) if not in_window(t, L - 1, 1, 16, 1024)]
        sc = []
        for t in toks:
            acc = np.float32(0)
            for c in range(d):  # fp32 multiply-add in order, rounded once per step
                acc = np.float32(np.float64(qf[n, c]) * np.float64(kf[n, t, c]) + np.float64(acc))
            sc.append(acc)
        order = np.lexsort((np.array(toks), -np.array(sc, np.float64)))
        ref = sorted(toks[o] for o in order[:top_k])
        np.testing.assert_array_equal(got[n, :len(ref)], ref)


def test_selection_avoids_the_window_and_counts(oracle_mod):
    g = synth.rng(804)
    B, Lcap, d = 4, 5000, 16
    q = synth.normal_bits(g, (B, d))
    k = synth.normal_bits(g, (B, Lcap, d))
    lens = [5000, 1200, 1024, 1]
    pk = oracle_mod.hi_page_keys(k, lens)
    sel = oracle_mod.hi_select(q, k, pk, lens, 1, 16, 1024, 8, 500)
    for n, L in enumerate(lens):
        chosen = sel[n][sel[n] >= 0]
        assert np.all(np.diff(chosen) > 0)
        assert not any(in_window(int(t), L - 1, 1, 16, 1024) for t in chosen)
        outside = sum(1 for p in range(L // 128) for r in range(128)
                      if not in_window(p * 128 + r, L - 1, 1, 16, 1024))
        assert len(chosen) == min(500, outside, 8 * 128)


def test_decode_limits(oracle_mod):
    """No dynamic token: the fixed window alone (the SSA decode). Every token
    selected: the window and the selection cover the whole causal prefix, so
    the decode is full causal attention (the block oracle's unbounded window)."""
    g = synth.rng(805)
    H, D, B = 4, 64, 2
    lens = [2000, 700]
    Lcap = max(lens)
    q = synth.normal_bits(g, (B, H, D))
    kv = synth.normal_bits(g, (B, Lcap, 1, D))
    none = np.full((B, 0), -1, np.int32)
    o0, l0 = oracle_mod.hi_decode(q, kv, lens, H, 1, 16, 1024, 0.125, none, d_v=D)
    r0, rl0 = oracle_mod.decode(q, kv, None, np.array(lens, np.int32), H, 1, 1, 16, 1024, 0.125, d_v=D)
    np.testing.assert_allclose(o0, r0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l0, rl0, rtol=0, atol=1e-12)
    k_idx = synth.normal_bits(g, (B, Lcap, 8))
    q_idx = synth.normal_bits(g, (B, 8))
    pk = oracle_mod.hi_page_keys(k_idx, lens)
    # every token outside the window lies in a whole page only if the lengths are multiples of 128;
    # the partial last page always lies inside the 1,024-token window here
    sel = oracle_mod.hi_select(q_idx, k_idx, pk, lens, 1, 16, 1024, 10 ** 6, Lcap)
    o1, l1 = oracle_mod.hi_decode(q, kv, lens, H, 1, 16, 1024, 0.125, sel, d_v=D)
    r1, rl1 = oracle_mod.decode(q, kv, None, np.array(lens, np.int32), H, 1, 128, 0, -1, 0.125, d_v=D)
    np.testing.assert_allclose(o1, r1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, rl1, rtol=0, atol=1e-12)


def test_decode_is_the_lse_merge_of_its_two_parts(oracle_mod):
    """The decode over window and selection equals the log-sum-exp merge of
    attention over the window alone and over the selection alone (the merge
    oracle, pinned separately): the two parts are disjoint."""
    g = synth.rng(806)
    H, D, B = 4, 64, 2
    lens = [3000, 2500]
    Lcap = max(lens)
    q = synth.normal_bits(g, (B, H, D))
    kv = synth.normal_bits(g, (B, Lcap, 1, D))
    k_idx = synth.normal_bits(g, (B, Lcap, 8))
    q_idx = synth.normal_bits(g, (B, 8))
    pk = oracle_mod.hi_page_keys(k_idx, lens)
    sel = oracle_mod.hi_select(q_idx, k_idx, pk, lens, 1, 16, 1024, 6, 200)
    o, l = oracle_mod.hi_decode(q, kv, lens, H, 1, 16, 1024, 0.125, sel, d_v=D)
    ow, lw = oracle_mod.hi_decode(q, kv, lens, H, 1, 16, 1024, 0.125, np.full((B, 0), -1, np.int32), d_v=D)
    # the selection alone: a window that selects nothing (no sinks, zero local blocks is not a window,
    # so take the attention over the selected keys directly)
    qf = synth.bits_to_f32(q).astype(np.float64)
    kf = synth.bits_to_f32(kv).astype(np.float64)[:, :, 0]
    for n in range(B):
        keys = sel[n][sel[n] >= 0]
        z = 0.125 * qf[n] @ kf[n, keys].T                       # [H, K]
        ls = np.log(np.exp(z - z.max(1, keepdims=True)).sum(1)) + z.max(1)
        os_ = np.exp(z - ls[:, None]) @ kf[n, keys, :D]
        m = np.maximum(lw[n], ls)
        wa, wb = np.exp(lw[n] - m), np.exp(ls - m)
        np.testing.assert_allclose(o[n], (wa[:, None] * ow[n] + wb[:, None] * os_) / (wa + wb)[:, None], atol=1e-12)
        np.testing.assert_allclose(l[n], m + np.log(wa + wb), atol=1e-12)


@pytest.mark.parametrize("win,sel", [((1, 0, 50), [0, 5, 77]), ((4, 1, 3), [31, 4, 200]), ((1, 16, 1024), [])])
def test_decode_brute_force_small(oracle_mod, win, sel):
    """Tiny case by brute force: the keys are the window's (token-distance
    form, written out) plus an explicit selection that includes token 0 when
    the window has no sinks; one numpy softmax over them."""
    b, s, l = win
    g = synth.rng(807)
    H, D, L = 3, 32, 300
    q = synth.normal_bits(g, (1, H, D))
    kv = synth.normal_bits(g, (1, L, 1, D))
    i = L - 1
    keys = sorted(set(t for t in range(L) if in_window(t, i, b, s, l)) | set(sel))
    assert len(keys) == len(set(t for t in range(L) if in_window(t, i, b, s, l))) + len(sel)  # disjoint
    qf = synth.bits_to_f32(q).astype(np.float64)[0]
    kf = synth.bits_to_f32(kv).astype(np.float64)[0, :, 0]
    z = 0.2 * qf @ kf[keys].T
    w = np.exp(z)
    o_ref = (w @ kf[keys, :D]) / w.sum(1, keepdims=True)
    lse_ref = np.log(w.sum(1))
    selected = np.array([sel], np.int32) if sel else np.full((1, 0), -1, np.int32)
    o, lse = oracle_mod.hi_decode(q, kv, [L], H, b, s, l, 0.2, selected, d_v=D)
    np.testing.assert_allclose(o[0], o_ref, atol=1e-12)
    np.testing.assert_allclose(lse[0], lse_ref, atol=1e-12)
