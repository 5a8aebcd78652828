"""Seeded synthetic inputs shared by the CUDA path, its tests and the oracle.

This module only draws numbers. It holds none of the paged-attention
arithmetic: no block tables, no slot mapping, no softmax, no allocator.
Both sides (the oracle under ``oracle/`` and the library under
``paged_kv_cache_358_b200/``) take the same arrays from here, so that a
parity test compares the two on identical inputs.

Random numbers come from ``numpy.random.Generator(PCG64(seed))``.  bf16
tensors are produced as their 16-bit patterns (``uint16``): a float32 draw
rounded to the nearest bf16, ties to even.  Both sides read those bits, so
the values are bit-identical on the host and on the device.

The workload shapes follow the five decode workloads of the pages:
  * tiny fp32 decode (lengths 37/91/128/201/511 plus edge lengths 0/1/16/17),
  * the 32-layer teaching model at 32 x 4096 history,
  * a 512-sequence mixed-length batch with a block-size sweep and scaled q,
  * prefix sharing with copy-on-write tails,
  * a large GQA 8:1 serving batch with lengths uniform on 1..8192.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

__all__ = [
    "rng",
    "normal_f32",
    "normal_bf16_bits",
    "bf16_bits_from_f32",
    "free_order",
    "uniform_lengths",
    "DecodeWorkload",
    "WORKLOADS",
    "workload",
]


def rng(seed: int) -> np.random.Generator:
    """The one generator every input is drawn from."""
    return np.random.Generator(np.random.PCG64(int(seed)))


def normal_f32(g: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    """float32 draws from N(0, 1), times ``scale`` (rounded once to f32)."""
    x = g.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x = (x * np.float32(scale)).astype(np.float32)
    return x


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bits.

    NaN inputs map to the canonical quiet NaN 0x7FC0.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out = out.copy()
        out[nan] = np.uint16(0x7FC0)
    return out


def normal_bf16_bits(g: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns of N(0, 1) draws times ``scale``."""
    return bf16_bits_from_f32(normal_f32(g, shape, scale))


def free_order(g: np.random.Generator, num_blocks: int) -> np.ndarray:
    """A seeded permutation of the physical block ids 0..num_blocks-1 (int32)."""
    return g.permutation(num_blocks).astype(np.int32)


def uniform_lengths(g: np.random.Generator, n: int, lo: int, hi: int) -> np.ndarray:
    """``n`` integer lengths uniform on [lo, hi], both ends included (int32)."""
    return g.integers(lo, hi + 1, size=n, dtype=np.int64).astype(np.int32)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Shape of one decode workload (all sizes in tokens / heads / elements)."""

    name: str
    layers: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                      # "bf16" or "f32": q, k, v storage type
    lengths: Sequence[int]          # history length per sequence before decode
    pool_blocks: int                # physical blocks per layer
    q_scale: float = 1.0            # q multiplied by this before rounding
    seed: int = 0

    @property
    def num_seqs(self) -> int:
        return len(self.lengths)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


def _pool_blocks_for(lengths: Sequence[int], block_size: int, extra_tokens: int,
                     headroom: float) -> int:
    need = sum(-(-(int(n) + extra_tokens) // block_size) for n in lengths)
    return int(math.ceil(need * headroom))


def workload(name: str, *, block_size: Optional[int] = None, decode_steps: int = 64,
             seed: Optional[int] = None) -> DecodeWorkload:
    """Build one of the named workloads.

    ``decode_steps`` sizes the pool headroom for appends; ``block_size``
    overrides the block size where the workload sweeps it.
    """
    if name == "tiny":
        return DecodeWorkload("tiny", 1, 8, 2, 64, 16, "f32", (37, 91, 128, 201, 511),
                              pool_blocks=64, seed=0 if seed is None else seed)
    if name == "tiny_edge":
        return DecodeWorkload("tiny_edge", 1, 8, 2, 64, 16, "f32", (0, 1, 16, 17),
                              pool_blocks=64, seed=0 if seed is None else seed)
    if name == "teaching_32x4096":
        lengths = (4096,) * 32
        # 16 GiB of history per 32 layers plus 10 %, and room for the appends.
        blocks = _pool_blocks_for(lengths, 16, decode_steps, 1.10)
        return DecodeWorkload("teaching_32x4096", 32, 32, 8, 128, 16, "bf16", lengths,
                              pool_blocks=blocks, seed=1 if seed is None else seed)
    if name == "mixed_512":
        B = 16 if block_size is None else block_size
        g = rng(2 if seed is None else seed)
        lengths = tuple(int(x) for x in uniform_lengths(g, 512, 1, 512))
        blocks = _pool_blocks_for(lengths, B, decode_steps, 1.10)
        return DecodeWorkload("mixed_512", 1, 32, 8, 128, B, "bf16", lengths,
                              pool_blocks=blocks, seed=2 if seed is None else seed)
    if name == "prefix_cow":
        # 64 groups x 4 branches share one prompt; lengths are the prompt length.
        lengths = (2008,) * 256
        blocks = 64 * (-(-2008 // 16)) + 256 * (-(-(256 + 16) // 16)) + 64
        return DecodeWorkload("prefix_cow", 24, 16, 4, 128, 16, "bf16", lengths,
                              pool_blocks=blocks, seed=3 if seed is None else seed)
    if name == "large_serving":
        g = rng(4 if seed is None else seed)
        lengths = tuple(int(x) for x in uniform_lengths(g, 256, 1, 8192))
        blocks = _pool_blocks_for(lengths, 16, decode_steps, 1.10)
        return DecodeWorkload("large_serving", 24, 32, 4, 128, 16, "bf16", lengths,
                              pool_blocks=blocks, seed=4 if seed is None else seed)
    raise KeyError(name)


WORKLOADS: List[str] = ["tiny", "tiny_edge", "teaching_32x4096", "mixed_512", "prefix_cow",
                        "large_serving"]


def kv_history(g: np.random.Generator, wl: DecodeWorkload, n_tokens: int,
               scale: float = 1.0) -> np.ndarray:
    """K or V values for ``n_tokens`` tokens: [n_tokens, H_kv, d] (bits or f32)."""
    shape = (n_tokens, wl.num_kv_heads, wl.head_dim)
    if wl.dtype == "bf16":
        return normal_bf16_bits(g, shape, scale)
    return normal_f32(g, shape, scale)


def queries(g: np.random.Generator, wl: DecodeWorkload) -> np.ndarray:
    """q for one decode step: [S, H_q, d] (bits or f32), times the workload's q scale."""
    shape = (wl.num_seqs, wl.num_q_heads, wl.head_dim)
    if wl.dtype == "bf16":
        return normal_bf16_bits(g, shape, wl.q_scale)
    return normal_f32(g, shape, wl.q_scale)
