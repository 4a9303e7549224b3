"""Host-side check of how the kernels cover a window with 128-token tiles
(no GPU): the tiles the prefill and dQ walk per query tile, the query tiles
the dK/dV owners and the sink tiles' far chunks walk per key tile, and the
per-element masks, restated from the kernels' tile rules, must together count
every visible (query, key) pair of the definition exactly once, for block
sizes from 1 to 512."""
import random

import pytest

T = 128


def lo(i, b, l):
    return max(0, (i // b - l + 1) * b)


def visible(i, t, b, s, l):
    return t <= i and (t < s * b or t >= lo(i, b, l))


def prefill_tiles(qb, b, s, l):
    """Key tiles of query tile qb: sink tiles, then the local ones."""
    sinks = min((s * b + T - 1) // T, qb + 1)
    local_lo = max(sinks, lo(qb * T, b, l) // T)
    return list(range(sinks)) + list(range(local_lo, qb + 1))


def local_end(k, b, l):
    """One past the last query tile that sees key tile k through the local window."""
    return (((k * T + T - 1) // b + l) * b - 1) // T + 1


def key_queries(t, i0, b, s, l):
    """Queries i0 .. i0+63 that see key t."""
    hi = 64 if t < s * b else (t // b + l) * b - i0
    return {q for q in range(64) if q >= t - i0 and q < hi}


CASES = [(1, 16, 1024, 1500), (1, 0, 300, 700), (64, 2, 14, 2000), (32, 3, 20, 1000), (256, 1, 3, 1300),
         (16, 5, 30, 900), (512, 1, 2, 1500), (2, 0, 1, 400), (128, 1, 7, 1100)]


@pytest.mark.parametrize("b,s,l,L", CASES)
def test_tiles_cover_every_visible_pair_once(b, s, l, L):
    nq = (L + T - 1) // T
    truth = {(i, t) for i in range(L) for t in range(i + 1) if visible(i, t, b, s, l)}
    by_q = {}
    for qb in range(nq):
        for kb in prefill_tiles(qb, b, s, l):
            for i in range(qb * T, min(L, qb * T + T)):
                for t in range(kb * T, min(L, kb * T + T)):
                    if visible(i, t, b, s, l):
                        by_q[(i, t)] = by_q.get((i, t), 0) + 1
    assert set(by_q) == truth and set(by_q.values()) == {1}
    chunk = 3  # a small far chunk, so that several chunks are exercised
    by_k = {}
    sink_tiles = (s * b + T - 1) // T
    for k in range(nq):
        ranges = [(k, min(nq, local_end(k, b, l)))]
        if k < sink_tiles:
            far = max(0, nq - local_end(k, b, l))
            ranges += [(local_end(k, b, l) + c * chunk, min(nq, local_end(k, b, l) + (c + 1) * chunk))
                       for c in range((far + chunk - 1) // chunk)]
        for j_lo, j_hi in ranges:
            for j in range(j_lo, j_hi):
                for t in range(k * T, min(L, k * T + T)):
                    for half in range(2):
                        i0 = j * T + 64 * half
                        for q in key_queries(t, i0, b, s, l):
                            if i0 + q < L:
                                by_k[(i0 + q, t)] = by_k.get((i0 + q, t), 0) + 1
    assert set(by_k) == truth and set(by_k.values()) == {1}
