"""B200 (sm_100a) streaming sparse attention of LongCat ZigZag Attention.

Python binding of the C ABI in ``include/loza_ssa.h``: argument marshalling
only. Every step of the computation runs in the CUDA kernels of
``libloza_ssa.so``; there is no CPU path. If the library is missing or cannot
be loaded, every call raises.

Tensors are torch CUDA tensors (PyTorch provides device memory and streams):
  q [T, H, d_qk], k [T, Hkv, d_qk], v [T, Hkv, d_v] bf16 (rows may be strided,
  heads and head dims contiguous); for the absorbed MLA layout pass the latent
  [T, 1, 576] as k and its first 512 columns (a view of the same storage) as v.
"""
from __future__ import annotations

import ctypes
import os

from ._build import LIB_PATH, build  # noqa: F401  (build is re-exported)

LOZA_UNBOUNDED = -1
LOZA_OP_PREFILL, LOZA_OP_DECODE, LOZA_OP_BACKWARD, LOZA_OP_PREFILL_HOST = 0, 1, 2, 3

_STATUS = {
    0: "LOZA_OK",
    -1: "LOZA_ERR_INVALID_ARG",
    -2: "LOZA_ERR_UNSUPPORTED",
    -3: "LOZA_ERR_WORKSPACE",
    -4: "LOZA_ERR_CUDA",
    -5: "LOZA_ERR_TIMEOUT",
}

# Every symbol include/loza_ssa.h declares.
EXPORTED = [
    "loza_ssa_workspace_size",
    "loza_ssa_prefill",
    "loza_ssa_prefill_host",
    "loza_ssa_decode",
    "loza_ssa_decode_noalloc",
    "loza_ssa_decode_paged",
    "loza_ssa_merge",
    "loza_ssa_mix",
    "loza_ssa_backward",
    "loza_status_string",
    "loza_device_status",
    "loza_launch_count",
    "loza_hi_page_keys",
    "loza_hi_workspace_size",
    "loza_hi_select",
    "loza_ssa_decode_selected",
    "loza_hi_decode",
    "loza_wait_selftest",
]


class LozaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)}")
        self.status = status


class Params(ctypes.Structure):
    """loza_ssa_params {block_size, n_sink, n_local, scale}."""
    _fields_ = [("block_size", ctypes.c_int32), ("n_sink", ctypes.c_int32),
                ("n_local", ctypes.c_int32), ("scale", ctypes.c_float)]

    def __init__(self, scale: float, block_size: int = 128, n_sink: int = 1, n_local: int = 7):
        super().__init__(block_size, n_sink, n_local, scale)


_lib = None
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded libloza_ssa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run block_sparse_streaming_b200.build() "
                               "(nvcc, sm_100a); there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        L.loza_ssa_workspace_size.restype = _sz
        L.loza_ssa_workspace_size.argtypes = [ctypes.c_int, _i32, _i64, _i32, _i32, _i32, _i32, _i32, Params]
        L.loza_ssa_prefill.restype = ctypes.c_int
        L.loza_ssa_prefill.argtypes = [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32,
                                       _i64, _i64, _i64, Params, _vp, _vp, _vp, _sz, _vp]
        L.loza_ssa_prefill_host.restype = ctypes.c_int
        L.loza_ssa_prefill_host.argtypes = [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32, Params,
                                            _vp, _vp, _vp, _sz, _vp]
        L.loza_ssa_decode.restype = ctypes.c_int
        L.loza_ssa_decode.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i64, _i64, _i32, _i32, _i32, _i32,
                                      Params, _vp, _vp, _vp, _sz, _vp]
        L.loza_ssa_decode_noalloc.restype = ctypes.c_int
        L.loza_ssa_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i64, _i64, _i32, _i32, _i32, _i32,
                                              Params, _vp, _vp, _vp]
        L.loza_ssa_backward.restype = ctypes.c_int
        L.loza_ssa_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
                                        _i32, _i32, Params, _vp, _vp, _vp, _vp, _sz, _vp]
        L.loza_ssa_decode_paged.restype = ctypes.c_int
        L.loza_ssa_decode_paged.argtypes = [_vp, _vp, _i32, _i64, _vp, _i32, _vp, _i32, _i32, _i32, Params, _vp, _vp,
                                            _vp, _sz, _vp]
        L.loza_ssa_merge.restype = ctypes.c_int
        L.loza_ssa_merge.argtypes = [_vp, _vp, _vp, _vp, _i64, _i32, _vp, _vp, _vp]
        L.loza_ssa_mix.restype = ctypes.c_int
        L.loza_ssa_mix.argtypes = [_vp, _vp, _i64, ctypes.c_float, _vp, _vp]
        L.loza_status_string.restype = ctypes.c_char_p
        L.loza_status_string.argtypes = [ctypes.c_int]
        L.loza_device_status.restype = ctypes.c_int
        L.loza_device_status.argtypes = [_vp]
        L.loza_launch_count.restype = ctypes.c_uint64
        L.loza_launch_count.argtypes = []
        L.loza_wait_selftest.restype = ctypes.c_int
        L.loza_wait_selftest.argtypes = [ctypes.c_uint32, _vp]
        L.loza_hi_page_keys.restype = ctypes.c_int
        L.loza_hi_page_keys.argtypes = [_vp, _i64, _i64, _vp, _i32, _i32, _i32, _vp, _vp]
        L.loza_hi_workspace_size.restype = _sz
        L.loza_hi_workspace_size.argtypes = [_i32, _i32, _i32, _i32, Params]
        L.loza_hi_select.restype = ctypes.c_int
        L.loza_hi_select.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp, _i32, _i32, _i32, Params, _i32, _i32, _vp, _vp,
                                     _sz, _vp]
        L.loza_ssa_decode_selected.restype = ctypes.c_int
        L.loza_ssa_decode_selected.argtypes = [_vp, _vp, _i64, _i64, _vp, _i32, _i32, Params, _vp, _i32, _vp, _vp,
                                               _vp, _sz, _vp]
        L.loza_hi_decode.restype = ctypes.c_int
        L.loza_hi_decode.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i32, _i32, _i32, Params,
                                     _i32, _i32, _vp, _vp, _vp, _sz, _vp]
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        raise LozaError(rc, what)


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _require(t, name, dtype=None, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def _row_tensor(t, name):
    """[rows, heads, dim] with heads/dim contiguous; returns its row stride."""
    if t.stride(2) != 1 or (t.shape[1] > 1 and t.stride(1) != t.shape[2]):
        raise ValueError(f"{name}: heads and head dim must be contiguous within a row")
    return t.stride(0)


def workspace_size(op, batch, total_tokens, max_seqlen, n_heads, n_kv_heads, d_qk, d_v, params: Params) -> int:
    return int(lib().loza_ssa_workspace_size(op, batch, total_tokens, max_seqlen, n_heads, n_kv_heads,
                                             d_qk, d_v, params))


def loza_ssa_prefill(q, k, v, cu_seqlens, max_seqlen: int, params: Params, out=None, lse=None,
                     workspace=None, stream=None):
    """SSA forward over a packed batch. Returns (out [T,H,d_v] bf16, lse [T,H] fp32)."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, torch.bfloat16, 3)
    _require(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, H, d_qk = q.shape
    Hkv, d_v = k.shape[1], v.shape[2]
    if out is None:
        out = torch.empty((T, H, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = workspace_size(LOZA_OP_PREFILL, cu_seqlens.numel() - 1, T, int(max_seqlen), H, Hkv, d_qk, d_v, params)
        if n:
            workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib().loza_ssa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), cu_seqlens.numel() - 1, T,
                                int(max_seqlen), H, Hkv, d_qk, d_v, _row_tensor(q, "q"), _row_tensor(k, "k"),
                                _row_tensor(v, "v"), params, _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                _stream_ptr(stream))
    _check(rc, "loza_ssa_prefill")
    return out, lse


def loza_ssa_prefill_host(q, k, v, params: Params, cu_seqlens=None, max_seqlen=None, out=None, lse=None,
                          workspace=None, stream=None):
    """Prefill of a packed batch from and to host memory (copies inside the call,
    overlapped with the kernels). q [T, H, d_qk], k [T, Hkv, d_qk], v [T, Hkv, d_v]:
    contiguous bf16 CPU tensors (pinned for overlap); absorbed MLA: pass the
    latent [T, 1, 576] as k and v (the same tensor, or its first 512 columns).
    cu_seqlens: host sequence offsets [0, ..., T] (a list, numpy array or CPU
    tensor; None = one sequence of T tokens). Returns (out [T, H, d_v] bf16,
    lse [T, H] fp32) as CPU tensors; they hold the results once `stream`
    (default: the current CUDA stream) has passed the call. The workspace is a
    CUDA uint8 tensor (allocated if None)."""
    import numpy as np
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.dim() != 3:
            raise TypeError(f"{n} must be a 3-D bf16 tensor")
    T, H, d_qk = q.shape
    Hkv, d_v = k.shape[1], v.shape[2]
    latent = v.data_ptr() == k.data_ptr()
    for t, n in ((q, "q"), (k, "k")) + (() if latent else ((v, "v"),)):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    if latent and v.stride(0) != k.stride(0):
        raise ValueError("a latent v must be a column slice of k")
    if cu_seqlens is None:
        cu_seqlens = [0, T]
    if isinstance(cu_seqlens, torch.Tensor):
        cu_seqlens = cu_seqlens.cpu().numpy()
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    if cu.ndim != 1 or cu.size < 2:
        raise ValueError("cu_seqlens needs at least two offsets")
    batch = cu.size - 1
    if max_seqlen is None:
        max_seqlen = max(1, int(np.max(np.diff(cu))))
    pin = q.device.type == "cpu" and q.is_pinned()
    if out is None:
        out = torch.empty((T, H, d_v), dtype=torch.bfloat16, device=q.device, pin_memory=pin)
    if lse is None:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device, pin_memory=pin)
    if not out.is_contiguous() or not lse.is_contiguous():
        raise ValueError("out and lse must be contiguous")
    if workspace is None:
        n = workspace_size(LOZA_OP_PREFILL_HOST, batch, T, int(max_seqlen), H, Hkv, d_qk, d_v, params)
        if n == 0:
            raise LozaError(-2, "loza_ssa_prefill_host")
        workspace = torch.empty(n, dtype=torch.uint8, device="cuda")
    _require(workspace, "workspace", torch.uint8)
    rc = lib().loza_ssa_prefill_host(_ptr(q), _ptr(k), _ptr(k if latent else v),
                                     cu.ctypes.data_as(ctypes.c_void_p), batch, T, int(max_seqlen), H, Hkv, d_qk,
                                     d_v, params, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                     _stream_ptr(stream))
    _check(rc, "loza_ssa_prefill_host")
    return out, lse


def loza_ssa_decode(q, k_cache, v_cache, seqlens, max_seqlen: int, params: Params, out=None, lse=None,
                    workspace=None, stream=None):
    """SSA decode. q [B,H,d_qk]; k_cache [B,Lcap,Hkv,d_qk] (row/batch strides taken from the
    tensor); v_cache None for the absorbed latent cache. Returns (out [B,H,d_v], lse [B,H])."""
    import torch
    _require(q, "q", torch.bfloat16, 3)
    _require(k_cache, "k_cache", torch.bfloat16, 4)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, H, d_qk = q.shape
    Hkv = k_cache.shape[2]
    d_v = v_cache.shape[3] if v_cache is not None else 512
    if k_cache.stride(3) != 1 or (Hkv > 1 and k_cache.stride(2) != d_qk):
        raise ValueError("k_cache: heads and head dim must be contiguous within a row")
    if out is None:
        out = torch.empty((B, H, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = workspace_size(LOZA_OP_DECODE, B, 0, int(max_seqlen), H, Hkv, d_qk, d_v, params)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().loza_ssa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, int(max_seqlen),
                               k_cache.stride(0), k_cache.stride(1), H, Hkv, d_qk, d_v, params, _ptr(out),
                               _ptr(lse), _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(rc, "loza_ssa_decode")
    return out, lse


def loza_ssa_decode_noalloc(q, k_cache, v_cache, seqlens, max_seqlen: int, params: Params, out, lse,
                            stream=None):
    """Decode for callers that cannot allocate device memory: like loza_ssa_decode,
    but the split-KV partials live in a fixed 16 MiB array inside the library, so
    nothing is allocated here either (out and lse must be given). Calls that can
    overlap on the GPU share that array and must not run concurrently."""
    import torch
    _require(q, "q", torch.bfloat16, 3)
    _require(k_cache, "k_cache", torch.bfloat16, 4)
    _require(seqlens, "seqlens", torch.int32, 1)
    _require(out, "out", torch.bfloat16, 3)
    _require(lse, "lse", torch.float32, 2)
    B, H, d_qk = q.shape
    Hkv = k_cache.shape[2]
    d_v = v_cache.shape[3] if v_cache is not None else 512
    rc = lib().loza_ssa_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, int(max_seqlen),
                                       k_cache.stride(0), k_cache.stride(1), H, Hkv, d_qk, d_v, params, _ptr(out),
                                       _ptr(lse), _stream_ptr(stream))
    _check(rc, "loza_ssa_decode_noalloc")
    return out, lse


def loza_ssa_backward(q, k, v, out, dout, lse, cu_seqlens, max_seqlen: int, params: Params, dq=None, dk=None,
                      dv=None, workspace=None, stream=None):
    """SSA backward. All of q, k, v, out, dout contiguous [T, heads, dim]. Returns (dq, dk, dv)."""
    import torch
    T, H, d_qk = q.shape
    Hkv, d_v = k.shape[1], v.shape[2]
    B = cu_seqlens.numel() - 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        n = workspace_size(LOZA_OP_BACKWARD, B, T, int(max_seqlen), H, Hkv, d_qk, d_v, params)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().loza_ssa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(cu_seqlens),
                                 B, T, int(max_seqlen), H, Hkv, d_qk, d_v, params, _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(rc, "loza_ssa_backward")
    return dq, dk, dv


def device_status(stream=None) -> int:
    """Synchronise and return the kernels' device status (0, or -5 after a timed-out wait)."""
    return int(lib().loza_device_status(_stream_ptr(stream)))


def launch_count() -> int:
    return int(lib().loza_launch_count())


def loza_ssa_merge(o_a, lse_a, o_b, lse_b, out=None, lse_out=None, stream=None):
    """Attention over the union of two disjoint key sets from two branches:
    o_* [..., d_v] bf16 contiguous, lse_* of shape o_*.shape[:-1] fp32 (natural
    log, -inf for a branch without keys). Returns (out, lse_out)."""
    import torch
    _require(o_a, "o_a", torch.bfloat16)
    _require(o_b, "o_b", torch.bfloat16)
    _require(lse_a, "lse_a", torch.float32)
    _require(lse_b, "lse_b", torch.float32)
    if o_a.shape != o_b.shape or lse_a.shape != o_a.shape[:-1] or lse_b.shape != o_a.shape[:-1]:
        raise ValueError("merge: branch shapes differ")
    for t, n in ((o_a, "o_a"), (o_b, "o_b"), (lse_a, "lse_a"), (lse_b, "lse_b")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    d_v = o_a.shape[-1]
    rows = o_a.numel() // d_v
    if out is None:
        out = torch.empty_like(o_a)
    if lse_out is None:
        lse_out = torch.empty_like(lse_a)
    rc = lib().loza_ssa_merge(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), rows, d_v, _ptr(out), _ptr(lse_out),
                              _stream_ptr(stream))
    _check(rc, "loza_ssa_merge")
    return out, lse_out


def loza_ssa_mix(o_full, o_ssa, alpha: float, out=None, stream=None):
    """alpha * o_full + (1 - alpha) * o_ssa (bf16, contiguous, same shape)."""
    import torch
    _require(o_full, "o_full", torch.bfloat16)
    _require(o_ssa, "o_ssa", torch.bfloat16)
    if o_full.shape != o_ssa.shape or not o_full.is_contiguous() or not o_ssa.is_contiguous():
        raise ValueError("mix: inputs must be contiguous and of one shape")
    if out is None:
        out = torch.empty_like(o_full)
    rc = lib().loza_ssa_mix(_ptr(o_full), _ptr(o_ssa), o_full.numel(), float(alpha), _ptr(out), _stream_ptr(stream))
    _check(rc, "loza_ssa_mix")
    return out


def loza_ssa_decode_paged(q, kv_pool, block_table, seqlens, max_seqlen: int, params: Params, out=None, lse=None,
                          workspace=None, stream=None):
    """Absorbed SSA decode from a paged latent cache. q [B,64,576]; kv_pool
    [num_pages, 128, 576] (or [num_pages * 128, 576]) bf16 with contiguous rows;
    block_table [B, pages per sequence] int32: the pool page of each logical
    128-token block. Returns (out [B,64,512], lse [B,64])."""
    import torch
    _require(q, "q", torch.bfloat16, 3)
    _require(kv_pool, "kv_pool", torch.bfloat16)
    _require(block_table, "block_table", torch.int32, 2)
    _require(seqlens, "seqlens", torch.int32, 1)
    if kv_pool.shape[-1] != 576 or kv_pool.stride(-1) != 1:
        raise ValueError("kv_pool rows must be 576 contiguous latent columns")
    pool2 = kv_pool.reshape(-1, 576) if kv_pool.dim() == 3 else kv_pool
    if pool2.dim() != 2 or pool2.shape[0] % 128 != 0:
        raise ValueError("kv_pool must hold whole pages of 128 rows")
    if not block_table.is_contiguous():
        raise ValueError("block_table must be contiguous")
    B, H, d_qk = q.shape
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = workspace_size(LOZA_OP_DECODE, B, 0, int(max_seqlen), H, 1, d_qk, 512, params)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().loza_ssa_decode_paged(_ptr(q), _ptr(pool2), pool2.shape[0] // 128, pool2.stride(0), _ptr(block_table),
                                     block_table.shape[1], _ptr(seqlens), B, int(max_seqlen), H, params, _ptr(out),
                                     _ptr(lse), _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(rc, "loza_ssa_decode_paged")
    return out, lse


# ---------------------------------------------------------------------------
# Hierarchical index decode (page 4's streaming-aware and hierarchical index)
# ---------------------------------------------------------------------------
def _contiguous(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _latent_cache(kv_cache):
    import torch
    _require(kv_cache, "kv_cache", torch.bfloat16, 4)
    if kv_cache.shape[2] != 1 or kv_cache.shape[3] < 576 or kv_cache.stride(3) != 1:
        raise ValueError("kv_cache must be [batch, rows, 1, 576] with contiguous latent rows")


def _index_keys(k_index):
    import torch
    _require(k_index, "k_index", torch.bfloat16, 3)
    if k_index.stride(2) != 1:
        raise ValueError("k_index: the index dimension must be contiguous")
    return k_index.shape[2], k_index.stride(0), k_index.stride(1)


def loza_hi_page_keys(k_index, seqlens, max_seqlen: int, page_keys=None, stream=None):
    """Mean index key of every whole 128-token page: k_index [B, Lcap, d] bf16 ->
    page_keys [B, d, max_seqlen // 128] float32 (pages innermost)."""
    import torch
    d, bs, rs = _index_keys(k_index)
    _require(seqlens, "seqlens", torch.int32, 1)
    B = k_index.shape[0]
    if page_keys is None:
        page_keys = torch.zeros((B, d, int(max_seqlen) // 128), dtype=torch.float32, device=k_index.device)
    _contiguous(page_keys, "page_keys")
    rc = lib().loza_hi_page_keys(_ptr(k_index), bs, rs, _ptr(seqlens), B, int(max_seqlen), d, _ptr(page_keys),
                                 _stream_ptr(stream))
    _check(rc, "loza_hi_page_keys")
    return page_keys


def hi_workspace_size(batch, max_seqlen, top_pages, top_k, params: Params) -> int:
    return int(lib().loza_hi_workspace_size(batch, max_seqlen, top_pages, top_k, params))


def loza_hi_select(q_index, k_index, page_keys, seqlens, max_seqlen: int, params: Params, top_pages: int, top_k: int,
                   selected=None, workspace=None, stream=None):
    """Tokens the hierarchical index selects: int32 [B, top_k], ascending, -1 padded."""
    import torch
    d, bs, rs = _index_keys(k_index)
    _require(q_index, "q_index", torch.bfloat16, 2)
    _require(page_keys, "page_keys", torch.float32, 3)
    _contiguous(q_index, "q_index")
    _contiguous(page_keys, "page_keys")
    B = k_index.shape[0]
    if selected is None:
        selected = torch.empty((B, top_k), dtype=torch.int32, device=k_index.device)
    if workspace is None:
        workspace = torch.empty(max(16, hi_workspace_size(B, int(max_seqlen), top_pages, top_k, params)),
                                dtype=torch.uint8, device=k_index.device)
    rc = lib().loza_hi_select(_ptr(q_index), _ptr(k_index), bs, rs, _ptr(page_keys), _ptr(seqlens), B,
                              int(max_seqlen), d, params, top_pages, top_k, _ptr(selected), _ptr(workspace),
                              workspace.numel(), _stream_ptr(stream))
    _check(rc, "loza_hi_select")
    return selected


def loza_ssa_decode_selected(q, kv_cache, seqlens, max_seqlen: int, params: Params, selected, out=None, lse=None,
                             workspace=None, stream=None):
    """Attention of each decode query over its window `params` and the tokens of
    `selected` (int32 [B, top_k]; entries that are negative, past the query or
    inside the window are ignored). Absorbed latent cache [B, Lcap, 1, 576];
    returns (out [B, 64, 512], lse [B, 64])."""
    import torch
    _require(q, "q", torch.bfloat16, 3)
    _latent_cache(kv_cache)
    _require(selected, "selected", torch.int32, 2)
    _require(seqlens, "seqlens", torch.int32, 1)
    _contiguous(q, "q")
    _contiguous(selected, "selected")
    B, H, _ = q.shape
    top_k = selected.shape[1]
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(16, hi_workspace_size(B, int(max_seqlen), 1, top_k, params)),
                                dtype=torch.uint8, device=q.device)
    rc = lib().loza_ssa_decode_selected(_ptr(q), _ptr(kv_cache), kv_cache.stride(0), kv_cache.stride(1),
                                        _ptr(seqlens), B, int(max_seqlen), params, _ptr(selected), top_k, _ptr(out),
                                        _ptr(lse), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    _check(rc, "loza_ssa_decode_selected")
    return out, lse


def loza_hi_decode(q, kv_cache, q_index, k_index, page_keys, seqlens, max_seqlen: int, params: Params,
                   top_pages: int, top_k: int, out=None, lse=None, workspace=None, stream=None):
    """Decode over the window `params` and the tokens the hierarchical index
    selects, merged; returns (out [B, 64, 512], lse [B, 64])."""
    import torch
    _require(q, "q", torch.bfloat16, 3)
    _latent_cache(kv_cache)
    d, bs, rs = _index_keys(k_index)
    _require(q_index, "q_index", torch.bfloat16, 2)
    _require(page_keys, "page_keys", torch.float32, 3)
    for t, name in ((q, "q"), (q_index, "q_index"), (page_keys, "page_keys")):
        _contiguous(t, name)
    B, H, _ = q.shape
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(16, hi_workspace_size(B, int(max_seqlen), top_pages, top_k, params)),
                                dtype=torch.uint8, device=q.device)
    rc = lib().loza_hi_decode(_ptr(q), _ptr(kv_cache), kv_cache.stride(0), kv_cache.stride(1), _ptr(q_index),
                              _ptr(k_index), bs, rs, _ptr(page_keys), _ptr(seqlens), B, int(max_seqlen), d, params,
                              top_pages, top_k, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                              _stream_ptr(stream))
    _check(rc, "loza_hi_decode")
    return out, lse


def wait_selftest(limit_us: int, stream=None) -> int:
    """Launch the bounded-wait self-test (a wait that nothing completes gives
    up after limit_us); returns the status of the following device-status
    read, LOZA_ERR_TIMEOUT (-5) when the bound works."""
    _check(lib().loza_wait_selftest(int(limit_us), _stream_ptr(stream)), "loza_wait_selftest")
    return device_status(stream)
