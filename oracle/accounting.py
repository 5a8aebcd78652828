"""Closed-form byte and slot accounting (oracle; test infrastructure only).

Every function restates one formula of the pages in exact integer (or
``fractions.Fraction``) arithmetic:

* KV bytes per token, two tensors (K and V) per layer:
  [P1] formula M_KV (section "1. KV是每个活动序列的持续状态" and the formula
  block after section 6); [P2] section "128 KiB：每新增一个位置的账单";
  [P3] section "3. 键值预算可以明确写出" and equation (1).
* Allocated slots A_B(n) = B*ceil(n/B) and tail waste W_B = A_B - n:
  [P1] formula A_B/W_B; [P2] sections "把浪费限制在尾块里" and
  "把“尾块浪费”算成可观测的数"; [P3] section 5 and equation (2).
* Position utilisation U = sum n_i / sum B*ceil(n_i/B): [P1] formula U and
  its worked example.
* Expected tail waste (B-1)/2 for lengths uniform on 1..kB: [P3] eq. (3).
* Pool capacity in blocks and in fixed-length requests: [P2] section
  "24 GiB 的 KV 池，能同时容纳多少请求？" and the exercise
  "8 GiB 池能容纳多少条 1,025-token 请求？".
* Swap time of a KV image over a link: [P2] section
  "腾出显存以后，还要付一次恢复成本".
"""
from __future__ import annotations

from fractions import Fraction
from typing import Iterable, Sequence, Tuple

KiB = 1 << 10
MiB = 1 << 20
GiB = 1 << 30


def ceil_div(a: int, b: int) -> int:
    if b <= 0:
        raise ValueError("divisor must be positive")
    return -(-int(a) // int(b))


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_scalar: int) -> int:
    """2 * L * H_kv * d * b: K and V of every layer for one token."""
    return 2 * layers * kv_heads * head_dim * bytes_per_scalar


def kv_bytes(lengths: Iterable[int], layers: int, kv_heads: int, head_dim: int,
             bytes_per_scalar: int) -> int:
    """Equation (1) of P3: bytes per token times the summed retained lengths."""
    return kv_bytes_per_token(layers, kv_heads, head_dim, bytes_per_scalar) * sum(int(t) for t in lengths)


def blocks_needed(n: int, block_size: int) -> int:
    """ceil(n / B) physical blocks for a sequence of n tokens (0 for n = 0)."""
    if n < 0:
        raise ValueError("negative length")
    return ceil_div(n, block_size)


def allocated_slots(n: int, block_size: int) -> int:
    """A_B(n) = B * ceil(n / B)."""
    return block_size * blocks_needed(n, block_size)


def tail_waste(n: int, block_size: int) -> int:
    """W_B(n) = A_B(n) - n: empty slots of the last block."""
    return allocated_slots(n, block_size) - n


def fixed_reservation_waste(n: int, max_len: int) -> int:
    """Waste of reserving max_len contiguous slots for an n-token request."""
    if n > max_len:
        raise ValueError("request longer than the reservation")
    return max_len - n


def waste_table(lengths: Sequence[int], block_size: int) -> Tuple[int, int, int, int]:
    """(useful tokens, blocks, allocated slots, tail waste) summed over lengths."""
    useful = sum(int(n) for n in lengths)
    blocks = sum(blocks_needed(n, block_size) for n in lengths)
    slots = sum(allocated_slots(n, block_size) for n in lengths)
    waste = sum(tail_waste(n, block_size) for n in lengths)
    return useful, blocks, slots, waste


def position_utilisation(lengths: Sequence[int], block_size: int) -> Fraction:
    """U = sum n_i / sum B*ceil(n_i/B) as an exact fraction."""
    useful, _, slots, _ = waste_table(lengths, block_size)
    return Fraction(useful, slots)


def fixed_utilisation(lengths: Sequence[int], max_len: int) -> Fraction:
    """Useful positions over a fixed max_len reservation per request."""
    return Fraction(sum(int(n) for n in lengths), max_len * len(lengths))


def tail_waste_bound(num_requests: int, block_size: int) -> int:
    """Equation (2) of P3: W_tail <= N (B - 1) for N non-empty requests."""
    return num_requests * (block_size - 1)


def expected_tail_waste(block_size: int) -> Fraction:
    """Equation (3) of P3: (B - 1) / 2 for lengths uniform on 1..kB."""
    return Fraction(block_size - 1, 2)


def mean_tail_waste_exact(block_size: int, max_len: int) -> Fraction:
    """Mean of W_B(n) over n = 1..max_len, enumerated (no closed form used)."""
    total = sum(tail_waste(n, block_size) for n in range(1, max_len + 1))
    return Fraction(total, max_len)


def mean_fixed_waste_exact(max_len: int) -> Fraction:
    """Mean of max_len - n over n = 1..max_len, enumerated."""
    return Fraction(sum(max_len - n for n in range(1, max_len + 1)), max_len)


def pool_blocks(pool_bytes: int, bytes_per_token: int, block_size: int) -> int:
    """Whole physical blocks that fit in a pool of pool_bytes."""
    return int(pool_bytes) // (int(bytes_per_token) * int(block_size))


def requests_that_fit(num_blocks: int, request_tokens: int, block_size: int) -> Tuple[int, int]:
    """(requests, blocks left) for fixed-length requests that share no blocks."""
    per = blocks_needed(request_tokens, block_size)
    return num_blocks // per, num_blocks % per


def swap_seconds(num_bytes: int, link_bytes_per_s: float) -> float:
    """Ideal one-way transfer time of num_bytes over a link."""
    return float(num_bytes) / float(link_bytes_per_s)


def decode_read_bytes(lengths: Sequence[int], bytes_per_token: int) -> int:
    """Lower bound on KV bytes one decode step reads: every history slot once."""
    return bytes_per_token * sum(int(n) for n in lengths)
