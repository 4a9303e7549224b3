"""fp64 CPU oracle for LoZA streaming sparse attention (SSA).

TEST INFRASTRUCTURE. This package is the plain, slow reference that the CUDA
library is checked against. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import it. It shares no
code with the CUDA library, and the library never imports it.

The arithmetic lives in ``ssa_ref.c`` (plain C, double precision, OpenMP over
rows); this module only compiles it with gcc and marshals numpy arrays. What it
computes is stated in the header of ``ssa_ref.c`` with the passages it follows
(Efficient Context Scaling with LongCat ZigZag Attention: page 1 section 01,
page 2 section 2.2, page 5), and for the token-granular variant, page 4's
streaming-aware index (a fixed set of sink tokens plus a sliding window).

Every array argument holding model values is a numpy ``uint16`` array of bf16
bit patterns; the C side widens each exactly to double.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssa_ref.c")
_SRC_HI = os.path.join(_HERE, "hi_ref.c")
_LIB_PATH = os.path.join(_HERE, "libssa_oracle.so")
_lib = None

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile ssa_ref.c into libssa_oracle.so next to it (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_HI))):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-ffp-contract=off",
                    "-o", tmp, _SRC, _SRC_HI, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.ssa_oracle_forward_rows.restype = ctypes.c_int
        lib.ssa_oracle_forward_rows.argtypes = [
            _u16p, _u16p, _u16p, _i32p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            _i64p, ctypes.c_int64, _f64p, _f64p]
        lib.ssa_oracle_forward_tokens_rows.restype = ctypes.c_int
        lib.ssa_oracle_forward_tokens_rows.argtypes = [
            _u16p, _u16p, _u16p, _i32p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
            _i64p, ctypes.c_int64, _f64p, _f64p]
        lib.ssa_oracle_decode.restype = ctypes.c_int
        lib.ssa_oracle_decode.argtypes = [
            _u16p, _u16p, _u16p, ctypes.c_int64, ctypes.c_int64, _i32p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            _f64p, _f64p]
        lib.ssa_oracle_backward_rows.restype = ctypes.c_int
        lib.ssa_oracle_backward_rows.argtypes = [
            _u16p, _u16p, _u16p, _u16p, _i32p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            _i64p, ctypes.c_int64, _i64p, ctypes.c_int64,
            _f64p, _f64p, _f64p]
        lib.ssa_oracle_merge.restype = ctypes.c_int
        lib.ssa_oracle_merge.argtypes = [_u16p, _f64p, _u16p, _f64p, ctypes.c_int64, ctypes.c_int, _f64p, _f64p]
        lib.ssa_oracle_mix.restype = ctypes.c_int
        lib.ssa_oracle_mix.argtypes = [_u16p, _u16p, ctypes.c_int64, ctypes.c_double, _f64p]
        _f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
        lib.hi_oracle_page_keys.restype = ctypes.c_int
        lib.hi_oracle_page_keys.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, _i32p, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int64, _f32p]
        lib.hi_oracle_select.restype = ctypes.c_int
        lib.hi_oracle_select.argtypes = [_u16p, _u16p, ctypes.c_int64, ctypes.c_int64, _f32p, ctypes.c_int64, _i32p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, _i32p]
        lib.hi_oracle_decode.restype = ctypes.c_int
        lib.hi_oracle_decode.argtypes = [_u16p, _u16p, ctypes.c_int64, ctypes.c_int64, _i32p, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_double, _i32p, ctypes.c_int, _f64p, _f64p]
        lib.ssa_oracle_visible_count.restype = ctypes.c_int64
        lib.ssa_oracle_visible_count.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        _lib = lib
    return _lib


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (numpy uint16)")
    return a


def forward(q, k, v, cu_seqlens, n_heads, n_kv_heads, block_size=128, n_sink=1,
            n_local=7, scale=1.0, rows=None):
    """O [R,H,d_v] and LSE [R,H] (float64) for the query rows ``rows`` (all rows
    when None). q [T,H,d_qk], k [T,Hkv,d_qk], v [T,Hkv,d_v] uint16 bf16 bits;
    cu_seqlens int32 [B+1]. ``n_local=-1`` means an unbounded local window."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T = int(cu[-1])
    d_qk, d_v = q.shape[-1], v.shape[-1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.zeros((len(rows), n_heads, d_v), np.float64)
    lse = np.zeros((len(rows), n_heads), np.float64)
    rc = _load().ssa_oracle_forward_rows(q, k, v, cu, len(cu) - 1, n_heads, n_kv_heads,
                                         d_qk, d_v, block_size, n_sink, n_local,
                                         float(scale), rows, len(rows), o, lse)
    if rc != 0:
        raise ValueError("oracle forward rejected its arguments")
    return o, lse


def forward_tokens(q, k, v, cu_seqlens, n_heads, n_kv_heads, sink_tokens=16, window_tokens=1024,
                   scale=1.0, rows=None):
    """Token-granular variant: query i sees the keys t <= i with t < sink_tokens
    or i - t < window_tokens (page 4: 16 sink tokens and a 1,024-token sliding
    window). Same arguments and results as forward() otherwise."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T = int(cu[-1])
    d_qk, d_v = q.shape[-1], v.shape[-1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.zeros((len(rows), n_heads, d_v), np.float64)
    lse = np.zeros((len(rows), n_heads), np.float64)
    rc = _load().ssa_oracle_forward_tokens_rows(q, k, v, cu, len(cu) - 1, n_heads, n_kv_heads, d_qk, d_v,
                                                int(sink_tokens), int(window_tokens), float(scale), rows,
                                                len(rows), o, lse)
    if rc != 0:
        raise ValueError("oracle forward (token window) rejected its arguments")
    return o, lse


def decode(q, k_cache, v_cache, seqlens, n_heads, n_kv_heads, block_size=128,
           n_sink=1, n_local=7, scale=1.0, d_v=None):
    """O [B,H,d_v], LSE [B,H] for one query per sequence (position L_n - 1).
    q [B,H,d_qk]; k_cache [B,Lcap,Hkv,d_qk]; v_cache [B,Lcap,Hkv,d_v], or None
    for an absorbed latent cache whose first ``d_v`` columns are V (the cache
    is then read in place, so a large, sparsely filled array is never copied)."""
    q, kc = _u16(q), _u16(k_cache)
    if v_cache is None:
        if d_v is None or n_kv_heads != 1:
            raise ValueError("a latent cache needs d_v and one kv head")
        vc, v_row = kc, kc.shape[-1]
    else:
        vc = _u16(v_cache)
        d_v, v_row = vc.shape[-1], vc.shape[-1] * n_kv_heads
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    B = q.shape[0]
    d_qk = q.shape[-1]
    o = np.zeros((B, n_heads, d_v), np.float64)
    lse = np.zeros((B, n_heads), np.float64)
    rc = _load().ssa_oracle_decode(q, kc, vc, kc.shape[1], v_row, sl, B, n_heads, n_kv_heads,
                                   d_qk, d_v, block_size, n_sink, n_local, float(scale),
                                   o, lse)
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return o, lse


def backward(q, k, v, dout, cu_seqlens, n_heads, n_kv_heads, block_size=128,
             n_sink=1, n_local=7, scale=1.0, q_rows=None, k_rows=None):
    """dQ [Rq,H,d_qk] for ``q_rows`` and dK [Rk,Hkv,d_qk], dV [Rk,Hkv,d_v] for
    ``k_rows`` (float64); None selects every row."""
    q, k, v, dout = _u16(q), _u16(k), _u16(v), _u16(dout)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T = int(cu[-1])
    d_qk, d_v = q.shape[-1], v.shape[-1]
    q_rows = np.arange(T, dtype=np.int64) if q_rows is None else np.ascontiguousarray(q_rows, dtype=np.int64)
    k_rows = np.arange(T, dtype=np.int64) if k_rows is None else np.ascontiguousarray(k_rows, dtype=np.int64)
    dq = np.zeros((len(q_rows), n_heads, d_qk), np.float64)
    dk = np.zeros((len(k_rows), n_kv_heads, d_qk), np.float64)
    dv = np.zeros((len(k_rows), n_kv_heads, d_v), np.float64)
    rc = _load().ssa_oracle_backward_rows(q, k, v, dout, cu, len(cu) - 1, n_heads,
                                          n_kv_heads, d_qk, d_v, block_size, n_sink,
                                          n_local, float(scale), q_rows, len(q_rows),
                                          k_rows, len(k_rows), dq, dk, dv)
    if rc != 0:
        raise ValueError("oracle backward rejected its arguments")
    return dq, dk, dv


def visible_count(i, block_size=128, n_sink=1, n_local=7) -> int:
    """|A(i)| under the oracle's block-index map."""
    return int(_load().ssa_oracle_visible_count(int(i), block_size, n_sink, n_local))


def merge(o_a, lse_a, o_b, lse_b):
    """Attention over the union of two disjoint key sets from the two branches'
    (O, LSE): O [rows, d_v] bf16 bits, LSE [rows] (natural log; -inf = no
    keys). Returns O [rows, d_v] and LSE [rows] as float64."""
    o_a, o_b = _u16(o_a), _u16(o_b)
    if o_a.shape != o_b.shape or o_a.ndim != 2:
        raise ValueError("merge takes two [rows, d_v] outputs of one shape")
    rows, d_v = o_a.shape
    la = np.ascontiguousarray(lse_a, dtype=np.float64).reshape(rows)
    lb = np.ascontiguousarray(lse_b, dtype=np.float64).reshape(rows)
    o = np.zeros((rows, d_v), np.float64)
    lse = np.zeros(rows, np.float64)
    if _load().ssa_oracle_merge(o_a, la, o_b, lb, rows, d_v, o, lse) != 0:
        raise ValueError("oracle merge rejected its arguments")
    return o, lse


def mix(o_full, o_ssa, alpha):
    """alpha * O_full + (1 - alpha) * O_ssa, elementwise, float64."""
    a, b = _u16(o_full), _u16(o_ssa)
    if a.shape != b.shape:
        raise ValueError("mix takes two outputs of one shape")
    o = np.zeros(a.shape, np.float64)
    if _load().ssa_oracle_mix(a.reshape(-1), b.reshape(-1), a.size, float(alpha), o.reshape(-1)) != 0:
        raise ValueError("oracle mix rejected its arguments")
    return o


# ---------------------------------------------------------------------------
# Hierarchical index (page 4: pages of 128 tokens, top pages, then top tokens)
# ---------------------------------------------------------------------------
HI_PAGE = 128


def hi_page_keys(k_index, seqlens):
    """Mean index key of every whole 128-token page: k_index [B, Lcap, d] bf16
    bits -> float32 [B, Lcap // 128, d] (pages past a sequence's end are 0)."""
    k = _u16(k_index)
    B, Lcap, d = k.shape
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    pages = Lcap // HI_PAGE
    out = np.zeros((B, pages, d), np.float32)
    if _load().hi_oracle_page_keys(k, Lcap * d, d, sl, B, d, pages, out) != 0:
        raise ValueError("oracle page keys rejected its arguments")
    return out


def hi_select(q_index, k_index, page_keys, seqlens, block_size, n_sink, n_local, top_pages, top_k):
    """Tokens chosen by the hierarchical index for each sequence's decode query:
    int32 [B, top_k], ascending, unused entries -1. q_index [B, d]; k_index
    [B, Lcap, d] bf16 bits; page_keys from hi_page_keys."""
    q, k = _u16(q_index), _u16(k_index)
    B, Lcap, d = k.shape
    pk = np.ascontiguousarray(page_keys, dtype=np.float32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    out = np.full((B, max(top_k, 1)), -1, np.int32)
    if _load().hi_oracle_select(q, k, Lcap * d, d, pk, pk.shape[1], sl, B, d, block_size, n_sink, n_local,
                                top_pages, top_k, out) != 0:
        raise ValueError("oracle select rejected its arguments")
    return out[:, :top_k]


def hi_decode(q, kv_cache, seqlens, n_heads, block_size, n_sink, n_local, scale, selected, d_v=512):
    """O [B, H, d_v], LSE [B, H] (float64) of each decode query over its fixed
    window and its selected tokens; kv_cache [B, Lcap, 1, d_qk] latent bits."""
    q, kv = _u16(q), _u16(kv_cache)
    B = q.shape[0]
    d_qk = q.shape[-1]
    Lcap = kv.shape[1]
    sel = np.ascontiguousarray(selected, dtype=np.int32).reshape(B, -1)
    top_k = sel.shape[1]
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    o = np.zeros((B, n_heads, d_v), np.float64)
    lse = np.zeros((B, n_heads), np.float64)
    if _load().hi_oracle_decode(q, kv, Lcap * kv.shape[-1], kv.shape[-1], sl, B, n_heads, d_qk, d_v, block_size,
                                n_sink, n_local, float(scale), sel if top_k else np.zeros((B, 1), np.int32),
                                top_k, o, lse) != 0:
        raise ValueError("oracle HI decode rejected its arguments")
    return o, lse
