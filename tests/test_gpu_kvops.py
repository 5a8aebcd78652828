"""Slot mapping, append and copy-on-write copy on the GPU against the oracle,
bit-exact (they move bits; nothing is rounded)."""
import numpy as np
import pytest

import workloads as W
from oracle import kvops
from oracle.allocator import RefAllocator
from tests.paged_batch import device_batch, host_batch, oracle_tables

pytestmark = pytest.mark.gpu


def _bits(t):
    import torch

    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy().view(np.uint32)


def _host_bits(x):
    return x if x.dtype == np.uint16 else np.ascontiguousarray(x, np.float32).view(np.uint32)


@pytest.mark.parametrize("name,B", [("tiny", 16), ("mixed_512", 4), ("mixed_512", 64)])
def test_tables_slots_and_append_bit_exact(name, B):
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl = W.workload(name, block_size=B) if name == "mixed_512" else W.workload(name)
    lengths = list(wl.lengths)[:64]
    hb = host_batch(wl, lengths=lengths)
    db = device_batch(hb)
    # tables: C++ allocator == oracle allocator
    ref_tables = oracle_tables(hb)
    dev_tables = db.tables.cpu().numpy()
    for i, t in enumerate(ref_tables):
        assert dev_tables[i, :len(t)].tolist() == t
    # slot mapping on the device == oracle slot mapping
    rows = np.concatenate([np.full(n, i, np.int32) for i, n in enumerate(lengths)])
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in lengths])
    pos[::7] = -1                                   # padding positions give -1
    slots = pkv.slot_mapping(db.tables, torch.from_numpy(pos).cuda(), B,
                             rows=torch.from_numpy(rows).cuda()).cpu().numpy()
    ref_slots = kvops.slot_mapping(ref_tables, rows, pos, B)
    assert np.array_equal(slots, ref_slots)
    # pools after append == oracle pools after scatter (unwritten slots keep the poison bits)
    dt = np.uint16 if wl.dtype == "bf16" else np.float32
    fill = np.uint16(0x7FC0) if wl.dtype == "bf16" else np.float32(np.nan)
    for pool_dev, hist in ((db.k_pool, hb.k_hist), (db.v_pool, hb.v_hist)):
        ref_pool = kvops.new_pool(wl.pool_blocks, B, wl.num_kv_heads, wl.head_dim, dt, fill)
        for i, t in enumerate(ref_tables):
            kvops.scatter_history(ref_pool, t, hist[i])
        got = _bits(pool_dev)
        want = _host_bits(ref_pool)
        if wl.dtype == "f32":       # torch NaN fill and numpy NaN may differ in payload
            nan_got = np.isnan(pool_dev.cpu().numpy())
            nan_want = np.isnan(ref_pool)
            assert np.array_equal(nan_got, nan_want)
            assert np.array_equal(got[~nan_got], want[~nan_want])
        else:
            assert np.array_equal(got, want)


def test_address_mapping_token_6_on_device():
    """Table [P5, P1, P7], B = 4: token 6 is written at block 1, offset 2."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    tables = torch.tensor([[5, 1, 7]], dtype=torch.int32, device="cuda")
    slots = pkv.slot_mapping(tables, torch.tensor([6], dtype=torch.int32, device="cuda"), 4)
    assert slots.tolist() == [1 * 4 + 2]
    kp = torch.zeros(8, 4, 1, 64, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    x = torch.arange(64, dtype=torch.bfloat16, device="cuda").view(1, 1, 64)
    pkv.kv_append(x, -x, slots, kp, vp)
    assert torch.equal(kp[1, 2, 0], x[0, 0]) and torch.equal(vp[1, 2, 0], -x[0, 0])
    assert int((kp != 0).sum()) == 63           # nothing else written


def test_cow_content_isolation_on_device():
    """Shared tail P3 = a,b,c; B copies into P8 and writes Y; A writes X in place; all layers."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    B, L = 4, 3
    order = [3, 8] + [b for b in range(10) if b not in (3, 8)]
    a = pkv.BlockAllocator(10, B, free_order=order)
    assert a.add_seq(0, 3) == 0 and a.fork(0, 1) == 0
    kps = [torch.full((10, B, 2, 64), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    vps = [torch.full_like(kps[0], float("nan")) for _ in range(L)]
    abc = torch.arange(3 * 2 * 64, dtype=torch.float32).view(3, 2, 64).to(torch.bfloat16).cuda()
    for kp, vp in zip(kps, vps):
        kp[3, :3] = abc
        vp[3, :3] = -abc
    rc, per, copies = a.append([1, 0])
    assert rc == 0 and copies == [(3, 8, 3)]
    pkv.block_copy(kps, vps, torch.tensor(copies, dtype=torch.int32, device="cuda"))
    tables, lens = a.fill_tables([1, 0], 1)
    t = torch.from_numpy(tables).cuda()
    slots = pkv.slot_mapping(t, torch.from_numpy(lens - 1).cuda(), B)
    assert slots.tolist() == [8 * 4 + 3, 3 * 4 + 3]
    X = torch.full((1, 2, 64), 24.0, dtype=torch.bfloat16, device="cuda")
    Y = torch.full((1, 2, 64), 25.0, dtype=torch.bfloat16, device="cuda")
    for kp, vp in zip(kps, vps):
        pkv.kv_append(torch.cat([Y, X]), torch.cat([-Y, -X]), slots, kp, vp)
        assert torch.equal(kp[3, :3], abc) and torch.equal(kp[8, :3], abc)
        assert torch.equal(kp[3, 3], X[0]) and torch.equal(kp[8, 3], Y[0])
        assert torch.equal(vp[8, :3], -abc) and torch.equal(vp[8, 3], -Y[0])
    assert a.check()


def test_random_block_copies_bit_exact():
    import torch

    import paged_kv_cache_358_b200 as pkv

    g = W.rng(77)
    N, B, H, D, L = 40, 16, 4, 128, 4
    pools_k = [W.normal_bf16_bits(g, (N, B, H, D)) for _ in range(L)]
    pools_v = [W.normal_bf16_bits(g, (N, B, H, D)) for _ in range(L)]
    perm = g.permutation(N)
    copies = [(int(perm[i]), int(perm[i + 20]), int(g.integers(0, B + 1))) for i in range(12)]
    copies += [(5, 5, 3), (-1, 3, 2), (2, N, 2), (1, 2, B + 1)]   # skipped: same, negative, out of range, too long
    dk = [torch.from_numpy(p.view(np.int16)).view(torch.bfloat16).cuda() for p in pools_k]
    dv = [torch.from_numpy(p.view(np.int16)).view(torch.bfloat16).cuda() for p in pools_v]
    pkv.block_copy(dk, dv, torch.tensor(copies, dtype=torch.int32, device="cuda"))
    valid = [c for c in copies[:12]]
    kvops.block_copy(pools_k + pools_v, valid)
    for got, want in zip(dk + dv, pools_k + pools_v):
        assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)


def test_append_skips_padding_and_out_of_range_slots():
    import torch

    import paged_kv_cache_358_b200 as pkv

    kp = torch.zeros(4, 8, 2, 64, dtype=torch.float32, device="cuda")
    vp = torch.zeros_like(kp)
    k = torch.ones(3, 2, 64, device="cuda")
    slots = torch.tensor([-1, 4 * 8, 5], dtype=torch.int64, device="cuda")
    pkv.kv_append(k, 2 * k, slots, kp, vp)
    assert int((kp != 0).sum()) == 2 * 64 and torch.all(kp[0, 5] == 1) and torch.all(vp[0, 5] == 2)


def test_append_rejects_bad_arguments():
    import torch

    import paged_kv_cache_358_b200 as pkv

    kp = torch.zeros(4, 8, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.ones(1, 2, 64, dtype=torch.bfloat16, device="cuda")
    s = torch.zeros(1, dtype=torch.int64, device="cuda")
    L = pkv.lib()
    rc = L.pkv_kv_append(k.data_ptr(), k.data_ptr(), s.data_ptr(), 1, kp.data_ptr(), kp.data_ptr(), 2, 64,
                         8, 4, 7, None)               # unknown dtype
    assert rc == pkv.Status.INVALID
    rc = L.pkv_kv_append(k.data_ptr() + 2, k.data_ptr(), s.data_ptr(), 1, kp.data_ptr(), kp.data_ptr(), 2,
                         64, 8, 4, 0, None)           # misaligned
    assert rc == pkv.Status.INVALID


def test_preempt_by_swap_round_trip():
    """Preempt a request: swap its blocks (every layer, K and V) to pinned host memory,
    release them, let another request overwrite the pool, re-admit it (new block ids)
    and swap back in; the KV bytes and the attention output are unchanged."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    L, N, B, Hkv, D, Hq = 3, 64, 16, 4, 128, 16
    g = W.rng(5)
    order = W.free_order(g, N)
    a = pkv.BlockAllocator(N, B, free_order=order)
    k_pools = [torch.from_numpy(W.normal_bf16_bits(g, (N, B, Hkv, D)).view(np.int16)).view(torch.bfloat16).cuda()
               for _ in range(L)]
    v_pools = [torch.from_numpy(W.normal_bf16_bits(g, (N, B, Hkv, D)).view(np.int16)).view(torch.bfloat16).cuda()
               for _ in range(L)]
    n = 300
    assert a.add_seq(7, n) == 0
    old = a.table(7)
    snap_k = [kp[old].clone() for kp in k_pools]
    snap_v = [vp[old].clone() for vp in v_pools]
    q = torch.from_numpy(W.normal_bf16_bits(g, (1, Hq, D)).view(np.int16)).view(torch.bfloat16).cuda()

    def attend(table):
        t = torch.tensor([table], dtype=torch.int32, device="cuda")
        ln = torch.tensor([n], dtype=torch.int32, device="cuda")
        return [pkv.paged_decode_attn(q, kp, vp, t, ln, 1 / np.sqrt(D), out_dtype=torch.float32)
                for kp, vp in zip(k_pools, v_pools)]

    before = attend(old)
    host = torch.empty(len(old) * L * 2 * B * Hkv * D, dtype=torch.bfloat16).pin_memory()
    pkv.swap_blocks(k_pools, v_pools, torch.tensor(old, dtype=torch.int32, device="cuda"), host, to_host=True)
    torch.cuda.synchronize()
    assert a.free_seq(7) == 0                       # preempted: blocks back to the pool
    assert a.add_seq(8, N * B) == 0                 # another request takes the whole pool
    for kp, vp in zip(k_pools, v_pools):
        kp.fill_(0.0)
        vp.fill_(0.0)
    assert a.free_seq(8) == 0
    assert a.add_seq(7, n) == 0                     # re-admitted: other block ids
    new = a.table(7)
    assert new != old
    pkv.swap_blocks(k_pools, v_pools, torch.tensor(new, dtype=torch.int32, device="cuda"), host, to_host=False)
    for l in range(L):
        assert torch.equal(k_pools[l][new].view(torch.int16), snap_k[l].view(torch.int16))
        assert torch.equal(v_pools[l][new].view(torch.int16), snap_v[l].view(torch.int16))
    after = attend(new)
    for x, y in zip(before, after):
        assert torch.equal(x, y)
    assert a.check()


def test_swap_500mib_time_against_the_pages_estimate():
    """Move 500 MiB of KV out and back and report the time next to the pages' analytic
    19.5 ms one way at 25 GiB/s (the measured link may be faster or slower)."""
    import json

    import torch

    import paged_kv_cache_358_b200 as pkv

    L, B, Hkv, D = 32, 16, 8, 128                    # 128 KiB per token, 2 MiB per block (all layers)
    nblk = 250                                       # 250 * 2 MiB = 500 MiB
    N = nblk + 8
    k_pools = [torch.zeros((N, B, Hkv, D), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    v_pools = [torch.zeros((N, B, Hkv, D), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    blocks = torch.arange(nblk, dtype=torch.int32, device="cuda")
    host = torch.empty(nblk * L * 2 * B * Hkv * D, dtype=torch.bfloat16).pin_memory()
    assert host.numel() * 2 == 500 * 2 ** 20
    times = {}
    for name, to_host in (("out", True), ("in", False)):
        pkv.swap_blocks(k_pools, v_pools, blocks, host, to_host=to_host)     # warm-up
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pkv.swap_blocks(k_pools, v_pools, blocks, host, to_host=to_host)
        e1.record()
        torch.cuda.synchronize()
        times[name] = e0.elapsed_time(e1)
    rec = {"mib": 500, "out_ms": times["out"], "in_ms": times["in"],
           "out_gib_per_s": 500 / 1024 / (times["out"] / 1000), "in_gib_per_s": 500 / 1024 / (times["in"] / 1000),
           "pages_one_way_ms_at_25_gib_per_s": 19.5}
    print("swap 500 MiB:", json.dumps(rec))
    assert times["out"] > 0 and times["in"] > 0
