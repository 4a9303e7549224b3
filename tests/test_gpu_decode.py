"""GPU parity of SSA decode against the fp64 oracle.

Decode runs the last token of each sequence against its KV cache. Cache rows
the window does not select are filled with NaN, so any out-of-window read
shows up as a non-finite or different output (the bounds check); the same call
with those rows zeroed must give bit-identical results.
"""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_lse, assert_close_o, from_dev, to_dev

pytestmark = pytest.mark.gpu

NAN_BF16 = np.uint16(0x7FC0)


@pytest.fixture(scope="module")
def bss():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_streaming_b200 as m
    m.build()
    return m


def selected_rows(L, b=128, s=1, l=7):
    """Cache rows the decode query (position L-1) may read: whole selected blocks."""
    j = (L - 1) // b
    if l < 0:
        blocks = range(j + 1)
    else:
        blocks = sorted(set(range(min(s, j + 1))) | set(range(max(0, j - l + 1), j + 1)))
    return np.concatenate([np.arange(kb * b, min((kb + 1) * b, L)) for kb in blocks])


def absorbed_case(bss, oracle_mod, seed, lens, Lcap, n_sink=1, n_local=7, poison=True, compare=True):
    """Absorbed MLA decode: 64 heads, latent cache [B, Lcap, 1, 576]. Only the rows
    the window selects carry seeded values; every other row is NaN (or zero)."""
    import torch
    H, D = 64, 576
    B = len(lens)
    g = synth.rng(seed)
    q = synth.normal_bits(g, (B, H, D))
    cache_dev = torch.full((B, Lcap, 1, D), float("nan") if poison else 0.0, dtype=torch.bfloat16, device="cuda")
    host = np.empty((B, Lcap, 1, D), np.uint16)          # lazily backed: only touched rows materialise
    for n, L in enumerate(lens):
        rows = selected_rows(L, 128, n_sink, n_local)
        vals = synth.normal_bits(g, (len(rows), 1, D))
        host[n, rows] = vals
        cache_dev[n, torch.from_numpy(rows).cuda()] = to_dev(vals)
    seqlens = np.array(lens, np.int32)
    scale = 1.0 / math.sqrt(192.0)
    params = bss.Params(scale, 128, n_sink, n_local)
    out, lse = bss.loza_ssa_decode(to_dev(q), cache_dev, None, torch.from_numpy(seqlens).cuda(), Lcap, params)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    res = (out.clone(), lse.clone())
    if compare:
        o_ref, lse_ref = oracle_mod.decode(q, host, None, seqlens, H, 1, 128, n_sink, n_local, scale, d_v=512)
        assert_close_o(from_dev(out), o_ref, "absorbed decode O")
        assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "absorbed decode LSE")
    del cache_dev
    return res


def test_absorbed_decode_small(bss, oracle_mod):
    absorbed_case(bss, oracle_mod, 61, [1, 127, 128, 129, 1000, 1024, 1025, 3000], 3072)


def test_absorbed_decode_nan_bounds_bitwise(bss, oracle_mod):
    lens = [5, 300, 2049, 4000]
    o1, l1 = absorbed_case(bss, oracle_mod, 62, lens, 4096, poison=True, compare=False)
    o2, l2 = absorbed_case(bss, oracle_mod, 62, lens, 4096, poison=False, compare=False)
    import torch
    assert torch.isfinite(o1.float()).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("batch", [20, 40, 80])
def test_absorbed_decode_split_plans(bss, oracle_mod, batch):
    """Batches whose plans are: 4 CTAs per sequence splitting its blocks (a
    cluster merging on chip by bulk copies), 2 CTAs splitting its heads (no
    merge), and 1 CTA per sequence. Some sequences are shorter than the
    window, so some block splits have no key block at all."""
    g = synth.rng(70 + batch)
    lens = g.integers(1, 6000, size=batch)
    lens[:4] = [1, 129, 700, 2049]
    absorbed_case(bss, oracle_mod, 71 + batch, lens.tolist(), 6144)


def test_absorbed_decode_half_block_boundaries(bss, oracle_mod):
    """Positions at and around the half-block boundaries of the own block (its
    second half present or not, full or partial), the sink block as the own
    block, and more splits (4 per sequence) than some sequences have half blocks."""
    lens = [1, 63, 64, 65, 100, 128, 129, 192, 193, 256, 1025, 1088, 1089]
    absorbed_case(bss, oracle_mod, 93, lens, 1152)


def test_absorbed_decode_wide_window_two_splits(bss, oracle_mod):
    """A 22-block window (s=2, l=20) on 40 sequences: two CTAs of a cluster
    split each sequence's blocks and merge on chip."""
    g = synth.rng(90)
    lens = g.integers(1, 4000, size=40)
    lens[:3] = [1, 300, 2817]
    absorbed_case(bss, oracle_mod, 91, lens.tolist(), 4096, n_sink=2, n_local=20)


def test_absorbed_dense_decode(bss, oracle_mod):
    absorbed_case(bss, oracle_mod, 63, [1, 700, 5000, 9000], 9216, n_sink=0, n_local=-1)


def test_absorbed_decode_workload3_full_size(bss, oracle_mod):
    """64 sequences, contexts uniform in [65536, 131072], cache [64, 131072, 576]."""
    w = synth.WORKLOADS[3]
    g = synth.rng(synth.workload_seed(3))
    lens = synth.uniform_lengths(g, w["batch"], w["ctx_lo"], w["ctx_hi"]).tolist()
    absorbed_case(bss, oracle_mod, synth.workload_seed(3) + 1, lens, w["ctx_hi"])


def test_absorbed_decode_1m_context(bss, oracle_mod):
    """Workload 4's decode at its stated size: 32 sequences of 1,048,576 tokens,
    cache [32, 1048576, 576] (38.7 GB; every row outside the windows is NaN)."""
    w = synth.WORKLOADS[4]
    absorbed_case(bss, oracle_mod, synth.workload_seed(4) + 2, [w["decode_ctx"]] * w["decode_batch"],
                  w["decode_ctx"])


@pytest.mark.parametrize("lens", [[1, 64, 129, 1000], [5000, 70001, 65536]])
def test_absorbed_decode_equals_last_prefill_row(bss, lens):
    """Decode of the last token equals the last row of the prefill over the same
    latent rows (the streaming pattern serves both phases: page 1 section 01),
    for the absorbed 576/512 shapes, on the GPU: each sequence's prefill, with
    the decode query as its last query row, against one batched decode call."""
    import torch
    H, D, DV = 64, 576, 512
    g = synth.rng(400 + len(lens))
    B, Lcap = len(lens), max(lens)
    qd = synth.normal_bits(g, (B, H, D))
    cache = torch.zeros((B, Lcap, 1, D), dtype=torch.bfloat16, device="cuda")
    for n, L in enumerate(lens):
        cache[n, :L] = to_dev(synth.normal_bits(g, (L, 1, D)))
    params = bss.Params(1.0 / math.sqrt(192.0))
    seqlens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out, lse = bss.loza_ssa_decode(to_dev(qd), cache, None, seqlens, Lcap, params)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    for n, L in enumerate(lens):
        q = torch.zeros((L, H, D), dtype=torch.bfloat16, device="cuda")
        q[L - 1] = to_dev(qd[n])
        lat = cache[n, :L].contiguous()
        cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
        po, pl = bss.loza_ssa_prefill(q, lat, lat[:, :, :DV], cu, L, params)
        torch.cuda.synchronize()
        assert_close_o(from_dev(po[L - 1]), from_dev(out[n]), f"absorbed decode vs prefill row, L={L}")
        assert_close_lse(pl[L - 1].cpu().numpy().astype(np.float64), lse[n].cpu().numpy().astype(np.float64),
                         f"absorbed decode vs prefill row LSE, L={L}")


@pytest.mark.parametrize("dqk,dv", [(64, 64), (192, 128)])
def test_mha_decode_matches_oracle_and_prefill(bss, oracle_mod, dqk, dv):
    """Per-head K/V decode; workload 1 shape for d = 64 (L = 2048, 4 heads, scale 1/8).
    Decode of the last token must also equal the last row of the prefill."""
    import torch
    H = 4
    lens = [2048] if dqk == 64 else [2048, 900, 1]
    B, Lcap = len(lens), max(lens)
    g = synth.rng(synth.workload_seed(1) + dqk)
    kc = synth.normal_bits(g, (B, Lcap, H, dqk))
    vc = synth.normal_bits(g, (B, Lcap, H, dv))
    qd = synth.normal_bits(g, (B, H, dqk))
    scale = 1 / 8 if dqk == 64 else 1 / math.sqrt(192)
    params = bss.Params(scale)
    seqlens = np.array(lens, np.int32)
    out, lse = bss.loza_ssa_decode(to_dev(qd), to_dev(kc), to_dev(vc), torch.from_numpy(seqlens).cuda(), Lcap,
                                   params)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.decode(qd, kc, vc, seqlens, H, H, 128, 1, 7, scale)
    assert_close_o(from_dev(out), o_ref, "mha decode O")
    assert_close_lse(lse.cpu().numpy().astype(np.float64), lse_ref, "mha decode LSE")
    # phase equivalence on the GPU: prefill with the decode query as the last row
    for n, L in enumerate(lens):
        q = np.zeros((L, H, dqk), np.uint16)
        q[L - 1] = qd[n]
        cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
        po, pl = bss.loza_ssa_prefill(to_dev(q), to_dev(kc[n, :L]), to_dev(vc[n, :L]), cu, L, params)
        torch.cuda.synchronize()
        assert_close_o(from_dev(po[L - 1]), from_dev(out[n]), "decode vs prefill row")
        assert abs(float(pl[L - 1, 0] - lse[n, 0])) <= 1e-3


def paged_case(bss, oracle_mod, seed, lens, n_sink=1, n_local=7):
    """Absorbed decode from a paged pool: each sequence's 128-token blocks sit
    on shuffled pages of a shared pool (unused pages hold NaN). Compared with
    the oracle on the logical cache, and bit for bit with loza_ssa_decode on a
    contiguous cache holding the same rows."""
    import torch
    H, D = 64, 576
    B = len(lens)
    g = synth.rng(seed)
    q = synth.normal_bits(g, (B, H, D))
    nblk = [(L + 127) // 128 for L in lens]
    n_pages = sum(nblk) + 5
    perm = g.permutation(n_pages)
    table = np.full((B, max(nblk) + 2), -1, np.int32)  # entries for absent blocks are never read
    Lcap = max(nblk) * 128
    pool = torch.full((n_pages, 128, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    cache = torch.full((B, Lcap, 1, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    host = np.empty((B, Lcap, 1, D), np.uint16)
    nxt = 0
    for n, L in enumerate(lens):
        for kb in range(nblk[n]):
            table[n, kb] = perm[nxt]
            nxt += 1
        rows = selected_rows(L, 128, n_sink, n_local)
        vals = synth.normal_bits(g, (len(rows), 1, D))
        host[n, rows] = vals
        dev_vals = to_dev(vals)
        cache[n, torch.from_numpy(rows).cuda()] = dev_vals
        pages = torch.from_numpy(table[n, rows // 128].astype(np.int64)).cuda()
        pool[pages, torch.from_numpy(rows % 128).cuda()] = dev_vals[:, 0]
    seqlens = torch.from_numpy(np.array(lens, np.int32)).cuda()
    scale = 1.0 / math.sqrt(192.0)
    params = bss.Params(scale, 128, n_sink, n_local)
    qd = to_dev(q)
    out_p, lse_p = bss.loza_ssa_decode_paged(qd, pool, torch.from_numpy(table).cuda(), seqlens, Lcap, params)
    out_c, lse_c = bss.loza_ssa_decode(qd, cache, None, seqlens, Lcap, params)
    torch.cuda.synchronize()
    assert bss.device_status() == 0
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
    o_ref, lse_ref = oracle_mod.decode(q, host, None, np.array(lens, np.int32), H, 1, 128, n_sink, n_local, scale,
                                       d_v=512)
    assert_close_o(from_dev(out_p), o_ref, "paged decode O")
    assert_close_lse(lse_p.cpu().numpy().astype(np.float64), lse_ref, "paged decode LSE")


@pytest.mark.parametrize("batch", [6, 40, 80])
def test_absorbed_decode_paged(bss, oracle_mod, batch):
    """Paged latent cache under the decode plans: half blocks split over a
    cluster of 4 CTAs (6 sequences) or 2 (40), and the block kernel with one CTA
    per sequence (80)."""
    g = synth.rng(300 + batch)
    lens = g.integers(1, 3000, size=batch)
    lens[:3] = [1, 128, 1025]
    paged_case(bss, oracle_mod, 301 + batch, lens.tolist())


def test_absorbed_decode_paged_wide_window_workspace_plan(bss, oracle_mod):
    """A 22-block window on 4 sequences: the plan keeps fp32 partials in the
    workspace and the last CTA of each sequence merges them; the cache is paged."""
    g = synth.rng(320)
    lens = g.integers(2000, 5000, size=4)
    lens[0] = 129
    paged_case(bss, oracle_mod, 321, lens.tolist(), n_sink=2, n_local=20)
