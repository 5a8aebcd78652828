"""Prefix cache on the device path: requests admitted through cached blocks
decode exactly as over their whole history.

[P2] "PagedAttention：让 KV cache 按需生长", section "请求结束，块就能交给下一位":
a released full block can stay in a cache with its content key; section
"只读时共用，要写入时再分开": a full-block hit is shared without a copy.  The
allocator (C++, through the binding) admits requests with the keys of their
leading full blocks; only the blocks that missed are written with kv_append;
every request is then decoded and compared with dense float64 attention over
its whole history (the hit blocks' contents were written by the request that
first held them).  The oracle allocator runs the same operations and must
agree on every status, hit count, table and the block states.

Content model: a keyed block holds a fixed content drawn from the key (two
requests whose leading keys agree hold the same tokens there); a block that
misses holds the request's own tokens.  Operations:
1. A, B, C admitted cold; their full blocks get keys.
2. D shares A's first three blocks while A is live, then misses.
3. A is released: its one block nobody else holds goes to the cached set.
4. E hits A's three live blocks and revives the cached one.
5. F hits one key, misses the second: later keys that exist are not used.
6. A request without keys fills the pool and evicts cached blocks; a request
   with an evicted key gets no hit there.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
from oracle.allocator import RefAllocator
from tests.paged_batch import as_f64, torch_from_host

pytestmark = pytest.mark.gpu

B, HQ, HKV, D = 16, 16, 4, 128
SCALE = 1.0 / np.sqrt(D)


def _key_content(key):
    g = W.rng(10_000 + key)
    return W.normal_bf16_bits(g, (B, HKV, D)), W.normal_bf16_bits(g, (B, HKV, D))


def test_prefix_cache_hits_decode_like_their_full_history():
    import torch

    import paged_kv_cache_358_b200 as pkv

    N = 40
    order = W.free_order(W.rng(77), N)
    cpp = pkv.BlockAllocator(N, B, free_order=order, enable_cache=True)
    ref = RefAllocator(N, B, free_order=order, enable_cache=True)
    kp = torch.full((N, B, HKV, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vp = torch.full_like(kp, float("nan"))
    own = W.rng(78)
    hist = {}     # request -> (K [n, H_kv, d], V) as the request sees its history

    def admit(sid, n, keys, expect_hits):
        r1 = ref.add_seq_prefix(sid, n, keys)
        r2 = cpp.add_seq_prefix(sid, n, keys)
        assert r1 == r2 == (0, expect_hits), (sid, r1, r2)
        nblk = -(-n // B)
        ks, vs = [], []
        for b in range(nblk):
            if b < len(keys):            # a keyed block holds the key's content
                kc, vc = _key_content(keys[b])
            else:                        # the request's own tokens
                kc, vc = W.normal_bf16_bits(own, (B, HKV, D)), W.normal_bf16_bits(own, (B, HKV, D))
            ks.append(kc)
            vs.append(vc)
        K = np.concatenate(ks)[:n]
        V = np.concatenate(vs)[:n]
        # write only the blocks that missed (positions expect_hits * B .. n - 1)
        start = expect_hits * B
        if start < n:
            tab, _ = cpp.fill_tables([sid], nblk)
            pos = torch.arange(start, n, dtype=torch.int32, device="cuda")
            slots = pkv.slot_mapping(torch.from_numpy(tab).cuda(), pos, B,
                                     rows=torch.zeros(n - start, dtype=torch.int32, device="cuda"))
            pkv.kv_append(torch_from_host(K[start:]), torch_from_host(V[start:]), slots, kp, vp)
        hist[sid] = (K, V)
        # publish the keys of the full blocks this request wrote, unless a key
        # already names another block
        for b in range(expect_hits, len(keys)):
            if keys[b] not in ref.block_of:
                assert ref.set_block_key(sid, b, keys[b]) == cpp.set_block_key(sid, b, keys[b]) == 0

    def release(sid):
        assert ref.free_seq(sid) == cpp.free_seq(sid) == 0
        hist.pop(sid)

    def same_state():
        live = sorted(hist)
        for sid in live:
            assert ref.table(sid) == cpp.table(sid)
            assert ref.length(sid) == cpp.length(sid)
        r_ref, r_free, r_cached = cpp.dump()
        assert r_ref == ref.ref and r_free == list(ref.free) and r_cached == list(ref.cached)
        assert ref.check() and cpp.check()

    def decode_all():
        live = sorted(hist)
        S = len(live)
        mb = max(len(ref.table(s)) for s in live)
        tables, lens = cpp.fill_tables(live, mb)
        g = W.rng(79 + S)
        q = W.normal_bf16_bits(g, (S, HQ, D))
        out = pkv.paged_decode_attn(torch_from_host(q), kp, vp, torch.from_numpy(tables).cuda(),
                                    torch.from_numpy(lens).cuda(), SCALE, out_dtype=torch.float32)
        got = as_f64(out)
        for i, sid in enumerate(live):
            K, V = hist[sid]
            assert int(lens[i]) == K.shape[0]
            exp = oatt.dense_decode(q[i], K, V, SCALE)
            assert np.max(np.abs(got[i] - exp)) <= 1e-2, sid

    a_keys = [101, 102, 103, 104]
    admit(0, 4 * B + 5, a_keys, 0)            # A: 4 full blocks + a partial tail
    admit(1, 2 * B + 3, [201, 202], 0)        # B
    admit(2, 3 * B, [301, 302, 303], 0)       # C
    same_state()
    admit(3, 4 * B + 9, a_keys[:3] + [401], 3)   # D: three live hits, then a miss
    same_state()
    decode_all()
    assert cpp.table(3)[:3] == cpp.table(0)[:3]
    release(0)                                 # A's fourth block (104) goes to the cached set
    st, rs = cpp.stats(), ref.stats()
    assert st["cached"] == rs["cached"] == 1
    assert (st["active"], st["free"]) == (rs["active"], rs["free"])
    admit(4, 5 * B + 1, a_keys + [501], 4)     # E: 3 live hits + the cached one revived
    assert cpp.stats()["cached"] == 0
    same_state()
    admit(5, 4 * B, [201, 999, 303], 1)        # F: one hit, then a miss; 303 exists but is not used
    assert cpp.table(5)[2] != cpp.table(2)[2]
    same_state()
    decode_all()
    # release B and C: their full blocks are cached with their keys
    release(1)
    release(2)
    same_state()
    cached_before = cpp.stats()["cached"]
    assert cached_before >= 4
    # a request without keys takes every free block and evicts cached ones
    free_now = cpp.stats()["free"]
    big = (free_now + 2) * B
    admit(6, big, [], 0)
    assert cpp.stats()["evictions"] == ref.stats()["evictions"] >= 2
    same_state()
    decode_all()
    # a key still in the cached set hits (nothing is allocated)
    r = ref.add_seq_prefix(7, B, [302])
    assert r == cpp.add_seq_prefix(7, B, [302]) == (0, 1)
    assert ref.free_seq(7) == cpp.free_seq(7) == 0
    # an evicted key no longer hits: the oldest cached blocks (B's 202, then C's 301) went first
    for sid, key in ((8, 202), (9, 301)):
        r = ref.add_seq_prefix(sid, B, [key])
        assert r == cpp.add_seq_prefix(sid, B, [key]) == (0, 0)
        assert ref.free_seq(sid) == cpp.free_seq(sid) == 0
    same_state()
