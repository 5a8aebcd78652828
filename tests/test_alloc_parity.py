"""The C++ host allocator against the oracle allocator, bit-exact.

Same seeded operation sequences go to both; after every operation the
statuses, copy lists, block tables, lengths, refcounts, free-queue order and
cached-set order must be identical, and both consistency checks must pass.
Also the printed walkthroughs of the pages run through the C++ allocator, and
host-side fault injection (forced allocation failure, skipped release) behaves
as specified.
"""
import random

import numpy as np
import pytest

import paged_kv_cache_358_b200 as pkv
from oracle.allocator import RefAllocator
from tests import test_oracle_pins as TP
from tests.conftest import golden


def _same(ref: RefAllocator, cpp: pkv.BlockAllocator, live):
    refc, free, cached = cpp.dump()
    assert refc == ref.ref
    assert free == list(ref.free)
    assert cached == list(ref.cached)
    for sid in live:
        assert cpp.table(sid) == ref.table(sid)
        assert cpp.length(sid) == ref.length(sid)
    st = cpp.stats()
    rs = ref.stats()
    for k in ("active", "cached", "free", "pool", "seqs", "allocs", "frees", "cow_copies",
              "alloc_failures", "evictions"):
        assert st[k] == rs[k], k
    assert cpp.check() and ref.check()


@pytest.mark.parametrize("seed,cache,B,N", [(0, False, 4, 64), (1, True, 4, 64), (2, False, 16, 200),
                                            (3, True, 16, 48), (4, False, 1, 32), (5, True, 8, 16)])
def test_random_sequences_bit_exact(seed, cache, B, N):
    rnd = random.Random(seed)
    order = rnd.sample(range(N), N)
    ref = RefAllocator(N, B, free_order=order, enable_cache=cache)
    cpp = pkv.BlockAllocator(N, B, free_order=order, enable_cache=cache)
    live, nxt = [], 0
    for step in range(1500):
        op = rnd.random()
        if op < 0.22 or not live:
            n = rnd.randint(0, 5 * B)
            a, b = ref.add_seq(nxt, n), cpp.add_seq(nxt, n)
            assert a == b
            if a == 0:
                live.append(nxt)
            nxt += 1
        elif op < 0.35:
            p = rnd.choice(live)
            a, b = ref.fork(p, nxt), cpp.fork(p, nxt)
            assert a == b
            if a == 0:
                live.append(nxt)
            nxt += 1
        elif op < 0.85:
            ids = rnd.sample(live, rnd.randint(1, len(live)))
            if rnd.random() < 0.05:
                ids = ids + ids[:1]          # a repeated id: INVALID on both, nothing changes
            assert ref.append(ids) == cpp.append(ids)
        elif op < 0.97:
            sid = live.pop(rnd.randrange(len(live)))
            assert ref.free_seq(sid) == cpp.free_seq(sid) == 0
        else:
            bogus = nxt + 1000
            assert ref.free_seq(bogus) == cpp.free_seq(bogus) == pkv.Status.INVALID
            assert ref.fork(bogus, nxt) == cpp.fork(bogus, nxt) == pkv.Status.INVALID
        _same(ref, cpp, live)


def test_walkthroughs_through_cpp(monkeypatch):
    """The printed walkthroughs, run against the C++ allocator through the same pins."""
    class Adapter(pkv.BlockAllocator):
        @property
        def ref(self):
            return self.dump()[0]

        @property
        def free(self):
            return self.dump()[1]

        @property
        def cached(self):
            return self.dump()[2]

        @property
        def seqs(self):
            return {}

        def available(self):
            st = self.stats()
            return st["free"] + st["cached"]

    monkeypatch.setattr(TP, "RefAllocator", Adapter)
    TP.test_cow_walkthrough()
    TP.test_cow_content_isolation()
    TP.test_append_across_block()
    TP.test_admission_three_of_four()
    TP.test_cow_allocation_failure_keeps_mapping()


def test_capacity_examples_through_cpp():
    c = golden("capacity.json")["pool_24gib"]
    a = pkv.BlockAllocator(c["blocks"], c["block_size"])
    for i in range(c["requests"]):
        assert a.add_seq(i, c["request_tokens"]) == 0
    snap = a.dump()
    assert a.stats()["free"] == c["blocks_left"]
    assert a.add_seq(999, c["request_tokens"]) == pkv.Status.NO_BLOCKS
    assert a.dump() == snap and a.check()
    d = golden("capacity.json")["pool_8gib"]
    b = pkv.BlockAllocator(d["blocks"], d["block_size"])
    for i in range(d["requests"]):
        assert b.add_seq(i, d["request_tokens"]) == 0
    assert b.stats()["free"] == d["blocks_left"]
    assert b.add_seq(999, d["request_tokens"]) == pkv.Status.NO_BLOCKS
    t = golden("capacity.json")["teaching_log"]
    c3 = pkv.BlockAllocator(t["pool"], 4, enable_cache=True)
    for i in range(100):
        assert c3.add_seq(i, 40) == 0
    for i in range(30):
        assert c3.free_seq(i) == 0
    st = c3.stats()
    assert (st["active"], st["cached"], st["free"]) == (t["active"], t["cached"], t["free"])
    assert c3.add_seq(1000, t["request_blocks"] * 4) == pkv.Status.NO_BLOCKS
    assert c3.check()


def test_fault_injection_alloc_fail_changes_nothing():
    a = pkv.BlockAllocator(16, 4)
    assert a.add_seq(0, 4) == 0
    snap = (a.dump(), a.table(0), a.length(0))
    a.inject_fault(pkv.FAULT_ALLOC_FAIL, 1)
    rc, per, copies = a.append([0])
    assert rc == pkv.Status.NO_BLOCKS and per == [pkv.Status.NO_BLOCKS] and copies == []
    assert (a.dump(), a.table(0), a.length(0)) == snap
    rc, per, copies = a.append([0])          # the fault is consumed: the next one succeeds
    assert rc == 0 and a.length(0) == 5
    a.inject_fault(pkv.FAULT_ALLOC_FAIL, 1)
    assert a.add_seq(1, 3) == pkv.Status.NO_BLOCKS and a.stats()["seqs"] == 1
    assert a.check()


def test_fault_injection_skipped_release_is_a_detected_leak():
    a = pkv.BlockAllocator(16, 4)
    for i in range(4):
        assert a.add_seq(i, 8) == 0
    a.inject_fault(pkv.FAULT_SKIP_RELEASE, 1)
    assert a.free_seq(0) == 0
    assert not a.check()                      # refcounts no longer match the live tables
    st = a.stats()
    assert st["active"] + st["cached"] + st["free"] == st["pool"]   # conservation alone misses it
    # cancelling the rest properly still leaves the leaked blocks unusable
    for i in range(1, 4):
        assert a.free_seq(i) == 0
    assert a.stats()["free"] == 14 and a.add_seq(9, 16 * 4) == pkv.Status.NO_BLOCKS


def test_fill_tables_and_errors():
    a = pkv.BlockAllocator(32, 4, free_order=list(range(31, -1, -1)))
    assert a.add_seq(5, 9) == 0 and a.add_seq(6, 0) == 0
    tables, lens = a.fill_tables([5, 6], 4, pad=-1)
    assert tables.tolist() == [[31, 30, 29, -1], [-1, -1, -1, -1]] and lens.tolist() == [9, 0]
    with pytest.raises(pkv.PkvError):
        a.fill_tables([5], 2)
    with pytest.raises(pkv.PkvError):
        a.fill_tables([7], 4)
    assert a.add_seq(5, 1) == pkv.Status.INVALID and a.add_seq(-1, 1) == pkv.Status.INVALID
    assert a.append([]) == (0, [], [])


@pytest.mark.parametrize("seed,cache", [(10, True), (11, False), (12, True)])
def test_prefix_cache_random_sequences_bit_exact(seed, cache):
    """Keys on full blocks, prefix admissions (hits on live and cached blocks), evictions."""
    rnd = random.Random(seed)
    N, B = 48, 4
    order = rnd.sample(range(N), N)
    ref = RefAllocator(N, B, free_order=order, enable_cache=cache)
    cpp = pkv.BlockAllocator(N, B, free_order=order, enable_cache=cache)
    live, nxt = [], 0
    prompts = {}      # seq -> list of block keys of its full blocks (prompt "tokens")
    for step in range(1500):
        op = rnd.random()
        if op < 0.25 or not live:
            # a prompt built from a few shared prefixes: keys chained like a content hash
            base = rnd.randint(0, 5)
            nfull = rnd.randint(0, 4)
            keys = [(base * 1000 + i) * 7919 for i in range(nfull)]
            n = nfull * B + rnd.randint(0, B)
            r1 = ref.add_seq_prefix(nxt, n, keys)
            r2 = cpp.add_seq_prefix(nxt, n, keys)
            assert r1 == r2
            if r1[0] == 0:
                live.append(nxt)
                prompts[nxt] = keys
                for i, k in enumerate(keys):            # publish the keys of its full blocks
                    a, b = ref.set_block_key(nxt, i, k), cpp.set_block_key(nxt, i, k)
                    assert a == b
            nxt += 1
        elif op < 0.35:
            sid = rnd.choice(live)
            lb = rnd.randint(0, 5)
            key = rnd.randint(0, 2 ** 64 - 1)
            assert ref.set_block_key(sid, lb, key) == cpp.set_block_key(sid, lb, key)
        elif op < 0.75:
            ids = rnd.sample(live, rnd.randint(1, len(live)))
            assert ref.append(ids) == cpp.append(ids)
        else:
            sid = live.pop(rnd.randrange(len(live)))
            assert ref.free_seq(sid) == cpp.free_seq(sid) == 0
        _same(ref, cpp, live)
        assert ref.stats()["prefix_hits"] == cpp.stats()["prefix_hits"]


def test_prefix_hit_revives_cached_block_and_eviction_forgets():
    """A released full block stays cached with its key; a later request with the same
    prefix reuses it without a copy; once evicted, the key no longer hits."""
    for A in (RefAllocator, pkv.BlockAllocator):
        a = A(4, 4, enable_cache=True)
        assert a.add_seq_prefix(0, 8, [111, 222]) == (0, 0)     # cold: no hits
        assert a.set_block_key(0, 0, 111) == 0 and a.set_block_key(0, 1, 222) == 0
        assert a.set_block_key(0, 1, 333) == 2                   # a block has one key
        t0 = a.table(0)
        assert a.free_seq(0) == 0
        st = a.stats()
        assert (st["active"], st["cached"], st["free"]) == (0, 2, 2)
        assert a.add_seq_prefix(1, 9, [111, 222]) == (0, 2)     # both blocks reused
        assert a.table(1)[:2] == t0
        st = a.stats()
        assert (st["active"], st["cached"], st["free"], st["prefix_hits"]) == (3, 0, 1, 2)
        assert a.add_seq_prefix(2, 8, [111, 999]) == (0, 1)     # live hit shares, miss stops
        assert a.table(2)[0] == t0[0] and a.check()
        assert a.free_seq(1) == 0 and a.free_seq(2) == 0
        # fill the pool so the cached blocks get evicted, then the keys miss
        assert a.add_seq(3, 16) == 0
        assert a.stats()["evictions"] >= 2
        assert a.free_seq(3) == 0
        assert a.add_seq_prefix(4, 4, [111]) == (0, 0)
        assert a.check()
