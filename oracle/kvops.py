"""Slot mapping, token append and block copy on NumPy pools (oracle).

Test infrastructure only.  Pools follow the teaching layout of [P2]
"PagedAttention：让 KV cache 按需生长", section "把 token 6 变成真正的内存地址":
one K pool and one V pool per layer, each ``[physical block, slot in block,
KV head, dim]``.  Logical token t of a request lives in logical block t // B
at offset t % B (section "读 token 6，先查表，再找偏移"); the block table gives
the physical block.  A "slot" is ``physical * B + offset``, i.e. the row of
the pool viewed as ``[blocks * B, H_kv, d]``.

Values are stored as they are given (bf16 as uint16 bit patterns, f32 as
float32), so append and copy compare bit-exactly.
"""
from __future__ import annotations

from typing import Iterable, Sequence, Tuple

import numpy as np


def logical_address(t: int, block_size: int) -> Tuple[int, int]:
    """(logical block, offset) of token t."""
    if t < 0:
        raise ValueError("negative position")
    return t // block_size, t % block_size


def slot_of(table: Sequence[int], t: int, block_size: int) -> int:
    """Slot of token t for a request whose block table is ``table``."""
    lb, off = logical_address(t, block_size)
    return int(table[lb]) * block_size + off


def slot_mapping(tables: Sequence[Sequence[int]], rows: Sequence[int], positions: Sequence[int],
                 block_size: int) -> np.ndarray:
    """int64 slot for each (row, position); a negative position maps to -1."""
    out = np.empty(len(positions), dtype=np.int64)
    for i, (r, p) in enumerate(zip(rows, positions)):
        out[i] = -1 if p < 0 else slot_of(tables[r], int(p), block_size)
    return out


def new_pool(num_blocks: int, block_size: int, kv_heads: int, head_dim: int, dtype,
             fill=0) -> np.ndarray:
    return np.full((num_blocks, block_size, kv_heads, head_dim), fill, dtype=dtype)


def append(pool: np.ndarray, slots: Sequence[int], x: np.ndarray) -> None:
    """Write x[i] (one token, all KV heads) into the given slot; slot < 0 is skipped."""
    nb, B = pool.shape[0], pool.shape[1]
    for i, s in enumerate(slots):
        s = int(s)
        if s < 0 or s >= nb * B:
            continue
        pool[s // B, s % B] = x[i]


def block_copy(pools: Iterable[np.ndarray], copies: Sequence[Tuple[int, int, int]]) -> None:
    """pool[dst, :n_valid] = pool[src, :n_valid] in every pool, copies in order."""
    for pool in pools:
        for src, dst, n_valid in copies:
            pool[dst, :n_valid] = pool[src, :n_valid].copy()


def gather_history(pool: np.ndarray, table: Sequence[int], length: int) -> np.ndarray:
    """Contiguous [length, H_kv, d] history of one request, read through its table."""
    B = pool.shape[1]
    if length == 0:
        return pool[:0, 0]
    rows = [pool[int(table[t // B]), t % B] for t in range(length)]
    return np.stack(rows, axis=0)


def scatter_history(pool: np.ndarray, table: Sequence[int], hist: np.ndarray) -> None:
    """Write a contiguous [n, H_kv, d] history into the pool through the table."""
    B = pool.shape[1]
    for t in range(hist.shape[0]):
        pool[int(table[t // B]), t % B] = hist[t]
