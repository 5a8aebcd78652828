"""Python binding of libpkv (paged KV-cache decode attention on B200).

Argument marshalling only: every step runs in the C-ABI library
``libpkv.so`` built from ``csrc/`` (CUDA kernels for sm_100a and the host
block allocator).  There is no fallback: if the library is missing, importing
the ops raises.  Names mirror the C entry points of ``include/pkv.h`` without
the ``pkv_`` prefix.  PyTorch supplies device memory and the current stream.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "lib", "library_path", "Status", "PkvError",
    "BF16", "F32",
    "decode_workspace_bytes", "paged_decode_attn", "decode_plan", "paged_decode_attn_run",
    "decode_status", "set_decode_kernel", "set_launch_overlap", "paged_decode_attn_append_run",
    "paged_attn_multi_query", "paged_decode_attn_shared_prefix", "shared_prefix_workspace",
    "kv_append", "block_copy", "slot_mapping", "swap_blocks",
    "BlockAllocator",
]

HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(HERE, "libpkv.so")

BF16 = 0
F32 = 1


class Status:
    OK = 0
    NO_BLOCKS = 1
    INVALID = 2
    CUDA = 3
    DEVICE_TIMEOUT = 4
    BAD_TABLE = 5
    PLAN_MISMATCH = 6


FAULT_NONE, FAULT_ALLOC_FAIL, FAULT_SKIP_RELEASE = 0, 1, 2


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = f"{what}: {lib().pkv_status_string(status).decode()} ({status})"
        if status == Status.CUDA:
            msg += f" [{lib().pkv_last_cuda_error().decode()}]"
        super().__init__(msg)
        self.status = status


class _Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("pool", "active", "cached", "free", "seqs", "allocs", "frees", "cow_copies",
                 "alloc_failures", "evictions", "prefix_hits")]


_LIB = None

_i32, _i64, _f32, _sz, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
_P32 = ctypes.POINTER(ctypes.c_int32)

_SIGS = {
    "pkv_version": (ctypes.c_char_p, []),
    "pkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pkv_last_cuda_error": (ctypes.c_char_p, []),
    "pkv_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "pkv_paged_decode_attn": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32,
                                             _i32, _f32, _i32, _vp, _i32, _vp, _sz, _vp]),
    "pkv_decode_plan": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "pkv_paged_decode_attn_run": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                                                 _i32, _i32, _f32, _i32, _vp, _i32, _vp, _sz, _vp]),
    "pkv_decode_status": (ctypes.c_int, [_vp, _vp]),
    "pkv_paged_decode_attn_append_run": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32,
                                                        _i32, _i32, _i32, _i32, _f32, _i32, _vp, _i32, _vp, _sz,
                                                        _vp]),
    "pkv_paged_decode_attn_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                                                     _i32, _i32, _f32, _i32, _vp, _i32, _vp]),
    "pkv_multi_query_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "pkv_paged_attn_multi_query": (ctypes.c_int, [_vp, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                                                  _i32, _i32, _f32, _i32, _vp, _i32, _vp, _sz, _vp]),
    "pkv_shared_prefix_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "pkv_paged_decode_attn_shared_prefix": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _i32,
                                                           _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp,
                                                           _i32, _vp, _sz, _vp]),
    "pkv_set_decode_kernel": (ctypes.c_int, [_i32]),
    "pkv_set_launch_overlap": (ctypes.c_int, [_i32]),
    "pkv_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_ulonglong, _vp, _sz, _vp]),
    "pkv_kv_append": (ctypes.c_int, [_vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_block_copy": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i32, _vp, _i32, _i32, _i32,
                                      _i32, _i32, _i32, _vp]),
    "pkv_slot_mapping": (ctypes.c_int, [_vp, _i32, _vp, _vp, _i32, _i32, _vp, _vp]),
    "pkv_swap_blocks": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i32, _vp, _i32, _vp, _i32, _i32,
                                       _i32, _i32, _i32, _i32, _vp]),
    "pkv_alloc_create": (_vp, [_i32, _i32, _P32, _i32]),
    "pkv_alloc_destroy": (None, [_vp]),
    "pkv_alloc_add_seq": (ctypes.c_int, [_vp, _i32, _i32]),
    "pkv_alloc_fork": (ctypes.c_int, [_vp, _i32, _i32]),
    "pkv_alloc_append": (ctypes.c_int, [_vp, _P32, _i32, _P32, _P32, _P32]),
    "pkv_alloc_free_seq": (ctypes.c_int, [_vp, _i32]),
    "pkv_alloc_get_table": (ctypes.c_int, [_vp, _i32, _P32, _i32, _P32, _P32]),
    "pkv_alloc_fill_tables": (ctypes.c_int, [_vp, _P32, _i32, _P32, _i32, _i32, _P32]),
    "pkv_alloc_stats": (ctypes.c_int, [_vp, ctypes.POINTER(_Stats)]),
    "pkv_alloc_check": (ctypes.c_int, [_vp]),
    "pkv_alloc_dump": (ctypes.c_int, [_vp, _P32, _P32, _P32, _P32, _P32]),
    "pkv_alloc_inject_fault": (ctypes.c_int, [_vp, _i32, _i32]),
    "pkv_alloc_set_block_key": (ctypes.c_int, [_vp, _i32, _i32, ctypes.c_uint64]),
    "pkv_alloc_add_seq_prefix": (ctypes.c_int, [_vp, _i32, _i32, ctypes.POINTER(ctypes.c_uint64), _i32, _P32]),
}


def lib() -> ctypes.CDLL:
    """Load libpkv.so (built in-tree); raise if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"{library_path} is not built; run __graft_entry__.build() "
                               "or python -m paged_kv_cache_358_b200.build")
        L = ctypes.CDLL(library_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(rc: int, what: str) -> None:
    if rc != Status.OK:
        raise PkvError(rc, what)


# -- torch marshalling ---------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int) -> int:
    n = lib().pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim)
    if n == 0:
        raise PkvError(Status.INVALID, "decode_workspace_bytes")
    return int(n)


def new_workspace(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int, device=None):
    torch = _torch()
    n = decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def _attn_args(q, k_pool, v_pool, block_tables, seq_lens, out):
    torch = _torch()
    S, Hq, D = q.shape
    N, B, Hkv, D2 = k_pool.shape
    if tuple(v_pool.shape) != tuple(k_pool.shape) or D2 != D:
        raise ValueError("k_pool/v_pool/q shapes disagree")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] < S or seq_lens.shape[0] < S:
        raise ValueError("block_tables must be [num_seqs, max_blocks]")
    if q.dtype != k_pool.dtype or v_pool.dtype != k_pool.dtype:
        raise TypeError("q, k_pool and v_pool must share a dtype")
    if tuple(out.shape) != (S, Hq, D):
        raise ValueError("out must be [num_seqs, num_q_heads, head_dim]")
    return S, Hq, Hkv, D, B, N


def paged_decode_attn(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out=None,
                      out_dtype=None, workspace=None, stream=None):
    """out[s, h] = softmax(scale * q[s, h] K^T) V over the paged history of request s."""
    torch = _torch()
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    S, Hq, Hkv, D, B, N = _attn_args(q, k_pool, v_pool, block_tables, seq_lens, out)
    if workspace is None:
        workspace = new_workspace(S, Hq, Hkv, D, q.device)
    rc = lib().pkv_paged_decode_attn(
        _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _dev(block_tables, "block_tables"),
        block_tables.shape[1], _dev(seq_lens, "seq_lens"), S, Hq, Hkv, D, B, N, float(scale),
        _dtype_code(k_pool), _dev(out, "out"), _dtype_code(out), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "paged_decode_attn")
    return out


def paged_attn_multi_query(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out=None,
                           out_dtype=None, workspace=None, stream=None):
    """q: [num_seqs, T, num_q_heads, head_dim]; query token i of request s sits at
    position seq_lens[s] - T + i and attends the paged history up to it (causal)."""
    torch = _torch()
    if q.dim() != 4:
        raise ValueError("q must be [num_seqs, num_q_tokens, num_q_heads, head_dim]")
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have the shape of q")
    S, T, Hq, D = q.shape
    _, _, Hkv, _, B, N = _attn_args(q[:, 0], k_pool, v_pool, block_tables, seq_lens, out[:, 0])
    if workspace is None:
        n = lib().pkv_multi_query_workspace_bytes(S, T, Hq, Hkv, D)
        if n == 0:
            raise PkvError(Status.INVALID, "multi_query_workspace_bytes")
        workspace = torch.zeros(int(n), dtype=torch.uint8, device=q.device)
    rc = lib().pkv_paged_attn_multi_query(
        _dev(q, "q"), T, _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _dev(block_tables, "block_tables"),
        block_tables.shape[1], _dev(seq_lens, "seq_lens"), S, Hq, Hkv, D, B, N, float(scale),
        _dtype_code(k_pool), _dev(out, "out"), _dtype_code(out), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "paged_attn_multi_query")
    return out


def shared_prefix_workspace(num_seqs: int, num_groups: int, max_group: int, num_q_heads: int,
                            num_kv_heads: int, head_dim: int, max_blocks: int, device=None):
    torch = _torch()
    n = lib().pkv_shared_prefix_workspace_bytes(num_seqs, num_groups, max_group, num_q_heads, num_kv_heads,
                                                head_dim, max_blocks)
    if n == 0:
        raise PkvError(Status.INVALID, "shared_prefix_workspace_bytes")
    return torch.zeros(int(n), dtype=torch.uint8, device=device or "cuda")


def paged_decode_attn_shared_prefix(q, k_pool, v_pool, block_tables, seq_lens, group_start, prefix_blocks,
                                    max_group: int, scale: float, out=None, out_dtype=None, workspace=None,
                                    stream=None):
    """Decode attention for groups of consecutive requests that share the first
    prefix_blocks[g] blocks of their tables; equal to paged_decode_attn."""
    torch = _torch()
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    S, Hq, Hkv, D, B, N = _attn_args(q, k_pool, v_pool, block_tables, seq_lens, out)
    if group_start.dtype != torch.int32 or prefix_blocks.dtype != torch.int32:
        raise TypeError("group_start and prefix_blocks must be int32")
    NG = prefix_blocks.shape[0]
    if group_start.shape[0] != NG + 1:
        raise ValueError("group_start must have num_groups + 1 entries")
    if workspace is None:
        workspace = shared_prefix_workspace(S, NG, max_group, Hq, Hkv, D, block_tables.shape[1], q.device)
    rc = lib().pkv_paged_decode_attn_shared_prefix(
        _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _dev(block_tables, "block_tables"),
        block_tables.shape[1], _dev(seq_lens, "seq_lens"), S, _dev(group_start, "group_start"),
        _dev(prefix_blocks, "prefix_blocks"), NG, int(max_group), Hq, Hkv, D, B, N, float(scale),
        _dtype_code(k_pool), _dev(out, "out"), _dtype_code(out), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "paged_decode_attn_shared_prefix")
    return out


def decode_plan(seq_lens, num_q_heads: int, num_kv_heads: int, head_dim: int, kv_dtype: int,
                workspace, num_seqs: Optional[int] = None, stream=None) -> None:
    S = seq_lens.shape[0] if num_seqs is None else num_seqs
    rc = lib().pkv_decode_plan(_dev(seq_lens, "seq_lens"), S, num_q_heads, num_kv_heads, head_dim,
                               kv_dtype, _dev(workspace, "workspace"),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "decode_plan")


def paged_decode_attn_run(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, workspace,
                          stream=None):
    S, Hq, Hkv, D, B, N = _attn_args(q, k_pool, v_pool, block_tables, seq_lens, out)
    rc = lib().pkv_paged_decode_attn_run(
        _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _dev(block_tables, "block_tables"),
        block_tables.shape[1], _dev(seq_lens, "seq_lens"), S, Hq, Hkv, D, B, N, float(scale),
        _dtype_code(k_pool), _dev(out, "out"), _dtype_code(out), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "paged_decode_attn_run")
    return out


def paged_decode_attn_append_run(q, k_new, v_new, slot_mapping, k_pool, v_pool, block_tables, seq_lens,
                                 scale: float, out, workspace, stream=None):
    """kv_append(k_new, v_new, slot_mapping) and paged_decode_attn_run in one launch (plan first)."""
    torch = _torch()
    S, Hq, Hkv, D, B, N = _attn_args(q, k_pool, v_pool, block_tables, seq_lens, out)
    if tuple(k_new.shape) != (S, Hkv, D) or tuple(v_new.shape) != (S, Hkv, D):
        raise ValueError("k_new/v_new must be [num_seqs, num_kv_heads, head_dim]")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape[0] < S:
        raise TypeError("slot_mapping must be int64 [num_seqs]")
    if k_new.dtype != k_pool.dtype or v_new.dtype != k_pool.dtype:
        raise TypeError("dtype mismatch")
    rc = lib().pkv_paged_decode_attn_append_run(
        _dev(q, "q"), _dev(k_new, "k_new"), _dev(v_new, "v_new"), _dev(slot_mapping, "slot_mapping"),
        _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _dev(block_tables, "block_tables"), block_tables.shape[1],
        _dev(seq_lens, "seq_lens"), S, Hq, Hkv, D, B, N, float(scale), _dtype_code(k_pool), _dev(out, "out"),
        _dtype_code(out), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc, "paged_decode_attn_append_run")
    return out


def decode_status(workspace, stream=None) -> int:
    """Synchronise and return (then clear) the device status word of a workspace."""
    return lib().pkv_decode_status(_dev(workspace, "workspace"), _stream(stream))


def set_decode_kernel(which: int) -> None:
    """0 automatic, 1 CUDA-core FMA tiles, 2 tensor-core tiles (bf16)."""
    _check(lib().pkv_set_decode_kernel(int(which)), "set_decode_kernel")


def set_launch_overlap(on: bool) -> None:
    """Programmatic dependent launch of the decode kernels (see pkv_set_launch_overlap)."""
    _check(lib().pkv_set_launch_overlap(1 if on else 0), "set_launch_overlap")


def kv_append(k, v, slot_mapping, k_pool, v_pool, stream=None) -> None:
    """pool[slot // B, slot % B] = k (and v) for each new token."""
    torch = _torch()
    n = k.shape[0]
    N, B, Hkv, D = k_pool.shape
    if tuple(k.shape) != (n, Hkv, D) or tuple(v.shape) != (n, Hkv, D):
        raise ValueError("k/v must be [n_tokens, num_kv_heads, head_dim]")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k.dtype != k_pool.dtype or v.dtype != k_pool.dtype or v_pool.dtype != k_pool.dtype:
        raise TypeError("dtype mismatch")
    rc = lib().pkv_kv_append(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping"), n,
                             _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), Hkv, D, B, N,
                             _dtype_code(k_pool), _stream(stream))
    _check(rc, "kv_append")


def block_copy(k_pools: Sequence, v_pools: Sequence, copies, stream=None) -> None:
    """Copy-on-write: pool[dst, :n_valid] = pool[src, :n_valid] for every layer's K and V."""
    torch = _torch()
    L = len(k_pools)
    if L != len(v_pools) or L == 0:
        raise ValueError("need the same number (>= 1) of K and V pools")
    if copies.dtype != torch.int32 or copies.dim() != 2 or copies.shape[1] != 3:
        raise TypeError("copies must be int32 [n, 3]")
    N, B, Hkv, D = k_pools[0].shape
    for p in list(k_pools) + list(v_pools):
        if tuple(p.shape) != (N, B, Hkv, D) or p.dtype != k_pools[0].dtype:
            raise ValueError("all pools must share shape and dtype")
    kp = (ctypes.c_void_p * L)(*[_dev(p, "k_pool").value for p in k_pools])
    vp = (ctypes.c_void_p * L)(*[_dev(p, "v_pool").value for p in v_pools])
    n = copies.shape[0]
    rc = lib().pkv_block_copy(kp, vp, L, _dev(copies, "copies") if n else None, n, Hkv, D, B, N,
                              _dtype_code(k_pools[0]), _stream(stream))
    _check(rc, "block_copy")


def swap_blocks(k_pools: Sequence, v_pools: Sequence, blocks, host_buf, to_host: bool, stream=None) -> None:
    """Move blocks (all layers, K and V) to / from a pinned host buffer [n][L][2][B][H_kv][d]."""
    torch = _torch()
    L = len(k_pools)
    if L != len(v_pools) or L == 0:
        raise ValueError("need the same number (>= 1) of K and V pools")
    N, B, Hkv, D = k_pools[0].shape
    if blocks.dtype != torch.int32 or blocks.dim() != 1:
        raise TypeError("blocks must be int32 [n]")
    n = blocks.shape[0]
    if host_buf.is_cuda or not host_buf.is_pinned() or not host_buf.is_contiguous():
        raise ValueError("host_buf must be contiguous pinned host memory")
    if host_buf.numel() * host_buf.element_size() < n * L * 2 * B * Hkv * D * k_pools[0].element_size():
        raise ValueError("host_buf too small")
    kp = (ctypes.c_void_p * L)(*[_dev(p, "k_pool").value for p in k_pools])
    vp = (ctypes.c_void_p * L)(*[_dev(p, "v_pool").value for p in v_pools])
    rc = lib().pkv_swap_blocks(kp, vp, L, _dev(blocks, "blocks") if n else None, n,
                               ctypes.c_void_p(host_buf.data_ptr()), int(bool(to_host)), Hkv, D, B, N,
                               _dtype_code(k_pools[0]), _stream(stream))
    _check(rc, "swap_blocks")


def slot_mapping(block_tables, positions, block_size: int, rows=None, out=None, stream=None):
    """slots[i] = table[rows[i]][positions[i] // B] * B + positions[i] % B (int64)."""
    torch = _torch()
    n = positions.shape[0]
    if out is None:
        out = torch.empty(n, dtype=torch.int64, device=positions.device)
    rc = lib().pkv_slot_mapping(_dev(block_tables, "block_tables"), block_tables.shape[1],
                                _dev(rows, "rows") if rows is not None else None,
                                _dev(positions, "positions"), n, block_size, _dev(out, "slots"),
                                _stream(stream))
    _check(rc, "slot_mapping")
    return out


# -- host allocator ------------------------------------------------------------
def _p32(a: np.ndarray):
    return a.ctypes.data_as(_P32)


class BlockAllocator:
    """Host block allocator (C++): FIFO free queue, refcounts, copy-on-write, allocate-or-fail."""

    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Sequence[int]] = None,
                 enable_cache: bool = False):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if self._order.shape != (self.num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
            order = _p32(self._order)
        h = lib().pkv_alloc_create(self.num_blocks, self.block_size, order, int(bool(enable_cache)))
        if not h:
            raise PkvError(Status.INVALID, "alloc_create")
        self._h = ctypes.c_void_p(h)

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().pkv_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int, n_tokens: int) -> int:
        return lib().pkv_alloc_add_seq(self._h, int(seq_id), int(n_tokens))

    def fork(self, parent: int, child: int) -> int:
        return lib().pkv_alloc_fork(self._h, int(parent), int(child))

    def append(self, seq_ids: Sequence[int]) -> Tuple[int, List[int], List[Tuple[int, int, int]]]:
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
        n = ids.shape[0]
        st = np.zeros(max(n, 1), dtype=np.int32)
        cp = np.zeros((max(n, 1), 3), dtype=np.int32)
        nc = np.zeros(1, dtype=np.int32)
        rc = lib().pkv_alloc_append(self._h, _p32(ids), n, _p32(st), _p32(cp), _p32(nc))
        if rc == Status.INVALID:
            return rc, [], []
        return rc, st[:n].tolist(), [tuple(int(x) for x in r) for r in cp[:nc[0]]]

    def append_arrays(self, seq_ids: np.ndarray, status: np.ndarray, copies: np.ndarray) -> Tuple[int, int]:
        """Allocation-free variant for hot loops: fills caller arrays, returns (rc, n_copies)."""
        nc = np.zeros(1, dtype=np.int32)
        rc = lib().pkv_alloc_append(self._h, _p32(seq_ids), seq_ids.shape[0], _p32(status), _p32(copies),
                                    _p32(nc))
        return rc, int(nc[0])

    def free_seq(self, seq_id: int) -> int:
        return lib().pkv_alloc_free_seq(self._h, int(seq_id))

    def table(self, seq_id: int) -> List[int]:
        n = np.zeros(1, dtype=np.int32)
        t = np.zeros(1, dtype=np.int32)
        _check(lib().pkv_alloc_get_table(self._h, int(seq_id), None, 0, _p32(n), _p32(t)), "get_table")
        out = np.zeros(max(int(n[0]), 1), dtype=np.int32)
        _check(lib().pkv_alloc_get_table(self._h, int(seq_id), _p32(out), out.shape[0], _p32(n), _p32(t)),
               "get_table")
        return out[:int(n[0])].tolist()

    def length(self, seq_id: int) -> int:
        n = np.zeros(1, dtype=np.int32)
        t = np.zeros(1, dtype=np.int32)
        _check(lib().pkv_alloc_get_table(self._h, int(seq_id), None, 0, _p32(n), _p32(t)), "get_table")
        return int(t[0])

    def fill_tables(self, seq_ids: Sequence[int], max_blocks: int, pad: int = 0,
                    tables: Optional[np.ndarray] = None, lens: Optional[np.ndarray] = None):
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
        n = ids.shape[0]
        if tables is None:
            tables = np.zeros((n, max_blocks), dtype=np.int32)
        if lens is None:
            lens = np.zeros(n, dtype=np.int32)
        _check(lib().pkv_alloc_fill_tables(self._h, _p32(ids), n, _p32(tables), int(max_blocks), int(pad),
                                           _p32(lens)), "fill_tables")
        return tables, lens

    def stats(self) -> dict:
        s = _Stats()
        _check(lib().pkv_alloc_stats(self._h, ctypes.byref(s)), "stats")
        return {n: int(getattr(s, n)) for n, _ in _Stats._fields_}

    def check(self) -> bool:
        return lib().pkv_alloc_check(self._h) == Status.OK

    def dump(self):
        N = max(self.num_blocks, 1)
        ref = np.zeros(N, dtype=np.int32)
        fr = np.zeros(N, dtype=np.int32)
        ca = np.zeros(N, dtype=np.int32)
        nf = np.zeros(1, dtype=np.int32)
        nc = np.zeros(1, dtype=np.int32)
        _check(lib().pkv_alloc_dump(self._h, _p32(ref), _p32(fr), _p32(nf), _p32(ca), _p32(nc)), "dump")
        return ref[:self.num_blocks].tolist(), fr[:nf[0]].tolist(), ca[:nc[0]].tolist()

    def set_block_key(self, seq_id: int, logical_block: int, key: int) -> int:
        return lib().pkv_alloc_set_block_key(self._h, int(seq_id), int(logical_block),
                                             ctypes.c_uint64(int(key) & 0xFFFFFFFFFFFFFFFF))

    def add_seq_prefix(self, seq_id: int, n_tokens: int, keys: Sequence[int]) -> Tuple[int, int]:
        k = np.ascontiguousarray(np.asarray([int(x) & 0xFFFFFFFFFFFFFFFF for x in keys], dtype=np.uint64))
        hit = np.zeros(1, dtype=np.int32)
        rc = lib().pkv_alloc_add_seq_prefix(self._h, int(seq_id), int(n_tokens),
                                            k.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)) if k.size else None,
                                            int(k.size), _p32(hit))
        return rc, int(hit[0])

    def inject_fault(self, kind: int, count: int = 1) -> None:
        _check(lib().pkv_alloc_inject_fault(self._h, int(kind), int(count)), "inject_fault")
