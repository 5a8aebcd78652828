"""Build one paged decode batch twice from the same seeded inputs: once through
the library (C++ allocator, device slot mapping and append) and once through
the oracle (reference allocator, NumPy pools, float64 attention).

Used by the GPU parity tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``.  Only the seeded draws (``workloads``) are shared.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np

import workloads as W
from oracle import attention as oatt
from oracle.allocator import RefAllocator


@dataclasses.dataclass
class HostBatch:
    wl: W.DecodeWorkload
    lengths: List[int]
    order: np.ndarray          # free-queue order (seeded permutation)
    k_hist: List[np.ndarray]   # per request [n, H_kv, d] (bf16 bits or f32)
    v_hist: List[np.ndarray]
    q: np.ndarray              # [S, H_q, d]


def host_batch(wl: W.DecodeWorkload, lengths: Optional[Sequence[int]] = None, seed: Optional[int] = None,
               q_scale: float = 1.0) -> HostBatch:
    g = W.rng(wl.seed if seed is None else seed)
    lengths = list(wl.lengths if lengths is None else lengths)
    order = W.free_order(g, wl.pool_blocks)
    k_hist = [W.kv_history(g, wl, n) for n in lengths]
    v_hist = [W.kv_history(g, wl, n) for n in lengths]
    shape = (len(lengths), wl.num_q_heads, wl.head_dim)
    if wl.dtype == "bf16":
        q = W.normal_bf16_bits(g, shape, q_scale)
    else:
        q = W.normal_f32(g, shape, q_scale)
    return HostBatch(wl, lengths, order, k_hist, v_hist, q)


def oracle_tables(hb: HostBatch) -> List[List[int]]:
    a = RefAllocator(hb.wl.pool_blocks, hb.wl.block_size, free_order=hb.order)
    for i, n in enumerate(hb.lengths):
        assert a.add_seq(i, n) == 0
    return [a.table(i) for i in range(len(hb.lengths))]


def oracle_out(hb: HostBatch, scale: Optional[float] = None, rows=None) -> np.ndarray:
    """Dense float64 reference for all (or the listed (s, h)) outputs."""
    sc = hb.wl.scale if scale is None else scale
    G = hb.wl.group
    if rows is None:
        return np.stack([oatt.dense_decode(hb.q[s], hb.k_hist[s], hb.v_hist[s], sc)
                         for s in range(len(hb.lengths))])
    out = []
    for s, h in rows:
        out.append(oatt.dense_decode_head(hb.q[s, h], hb.k_hist[s][:, h // G], hb.v_hist[s][:, h // G], sc))
    return np.stack(out)


# -- device side ---------------------------------------------------------------
def torch_from_host(x: np.ndarray, device="cuda"):
    import torch

    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


@dataclasses.dataclass
class DeviceBatch:
    alloc: object
    k_pool: object
    v_pool: object
    tables: object       # int32 [S, max_blocks] on device
    seq_lens: object     # int32 [S] on device
    q: object
    max_blocks: int


def device_batch(hb: HostBatch, max_blocks: Optional[int] = None, poison: bool = True,
                 layers: int = 1) -> DeviceBatch:
    """Admit every request in the C++ allocator and write its history with kv_append."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl = hb.wl
    B = wl.block_size
    a = pkv.BlockAllocator(wl.pool_blocks, B, free_order=hb.order)
    for i, n in enumerate(hb.lengths):
        rc = a.add_seq(i, n)
        if rc != 0:
            raise RuntimeError(f"pool too small for request {i} ({n} tokens)")
    mb = max_blocks or max(1, max(-(-n // B) for n in hb.lengths))
    tables, lens = a.fill_tables(list(range(len(hb.lengths))), mb, pad=0)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    shape = (wl.pool_blocks, B, wl.num_kv_heads, wl.head_dim)
    k_pool = torch.full(shape, float("nan") if poison else 0.0, dtype=dt, device="cuda")
    v_pool = torch.full(shape, float("nan") if poison else 0.0, dtype=dt, device="cuda")
    t_dev = torch.from_numpy(tables).cuda()
    l_dev = torch.from_numpy(lens).cuda()
    rows = np.concatenate([np.full(n, i, np.int32) for i, n in enumerate(hb.lengths)] + [np.zeros(0, np.int32)])
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in hb.lengths] + [np.zeros(0, np.int32)])
    if rows.size:
        slots = pkv.slot_mapping(t_dev, torch.from_numpy(pos).cuda(), B, rows=torch.from_numpy(rows).cuda())
        # write in chunks to bound the staging memory
        start = 0
        for i, n in enumerate(hb.lengths):
            if n == 0:
                continue
            k = torch_from_host(hb.k_hist[i])
            v = torch_from_host(hb.v_hist[i])
            pkv.kv_append(k, v, slots[start:start + n], k_pool, v_pool)
            start += n
    q = torch_from_host(hb.q)
    return DeviceBatch(a, k_pool, v_pool, t_dev, l_dev, q, mb)


def as_f64(t) -> np.ndarray:
    import torch

    return t.detach().to(torch.float64).cpu().numpy()


def bf16_out_tol(ref: np.ndarray, base: float) -> np.ndarray:
    """Tolerance for a bf16 output: the fp32 budget plus half a bf16 ulp of the value."""
    return base + np.abs(ref) * 2.0 ** -8
