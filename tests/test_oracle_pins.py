"""The oracle's accounting and allocator against the values the pages print.

Every expected number here comes from a fixture under tests/golden/ (typed in
from the pages, each with its citation) or from an exact closed form.
"""
from fractions import Fraction

import pytest

from oracle import accounting as acc
from oracle.allocator import INVALID, NO_BLOCKS, OK, RefAllocator
from oracle import kvops
from tests.conftest import golden

GiB, MiB, KiB = acc.GiB, acc.MiB, acc.KiB


# -- byte accounting ----------------------------------------------------------
def test_bytes_per_token():
    g = golden("bytes_per_token.json")
    for c in g["cases"]:
        assert acc.kv_bytes_per_token(c["layers"], c["kv_heads"], c["head_dim"], c["bytes"]) == c["bytes_per_token"], c["cite"]
    for c in g["request_bytes"]:
        b = acc.kv_bytes([c["tokens"]], c["layers"], c["kv_heads"], c["head_dim"], c["bytes"])
        assert Fraction(b, GiB) == Fraction(c["gib"]).limit_denominator(), c["cite"]
    d = g["decode_read"]
    assert acc.decode_read_bytes([d["history"]] * d["requests"], d["bytes_per_token"]) == d["gib"] * GiB


def test_witness_bytes_per_token():
    w = golden("witness.json")
    assert acc.kv_bytes_per_token(32, 8, 128, 2) == w["bytes_per_token"]


# -- slots and tail waste -----------------------------------------------------
def test_length_10_block_4():
    c = golden("waste_tables.json")["length_10"]
    assert acc.blocks_needed(c["length"], c["block_size"]) == c["blocks"]
    assert acc.allocated_slots(c["length"], c["block_size"]) == c["slots"]
    assert acc.tail_waste(c["length"], c["block_size"]) == c["empty"]


def test_b16_table_rows():
    t = golden("waste_tables.json")["b16_rows"]
    B = t["block_size"]
    for r in t["rows"]:
        assert acc.blocks_needed(r["length"], B) == r["blocks"]
        assert acc.allocated_slots(r["length"], B) == r["slots"]
        assert acc.tail_waste(r["length"], B) == r["waste"]
    useful, blocks, slots, waste = acc.waste_table([r["length"] for r in t["rows"]], B)
    assert (useful, blocks, slots, waste) == (t["total"]["useful"], t["total"]["blocks"],
                                              t["total"]["slots"], t["total"]["waste"])


def test_block_size_sweep():
    t = golden("waste_tables.json")["sweep"]
    for col in t["columns"]:
        _, blocks, slots, waste = acc.waste_table(t["lengths"], col["block_size"])
        assert (blocks, slots, waste) == (col["blocks"], col["slots"], col["empty"])
        assert Fraction(waste * t["bytes_per_token"], MiB) == Fraction(col["empty_mib"]).limit_denominator()


def test_lab_script_outputs():
    t = golden("waste_tables.json")["lab"]
    for run in t["runs"]:
        useful, blocks, slots, waste = acc.waste_table(t["lengths"], run["block_size"])
        assert blocks == run["blocks"] and waste == run["tail_waste"]
        if "slots" in run:
            assert slots == run["slots"] and useful == run["useful"]


def test_position_utilisation():
    u = golden("utilisation.json")
    L = u["lengths"]
    assert sum(L) == u["useful"]
    assert u["fixed_reservation"] * len(L) == u["slots"]["fixed_512"]
    assert acc.waste_table(L, 16)[2] == u["slots"]["paged_16"]
    assert acc.waste_table(L, 32)[2] == u["slots"]["paged_32"]
    nd = u["printed_decimals"]
    assert round(float(acc.fixed_utilisation(L, 512)) * 100, nd) == u["utilisation_percent"]["fixed_512"]
    assert round(float(acc.position_utilisation(L, 16)) * 100, nd) == u["utilisation_percent"]["paged_16"]
    assert round(float(acc.position_utilisation(L, 32)) * 100, nd) == u["utilisation_percent"]["paged_32"]


def test_tail_waste_expectation_and_bound():
    t = golden("tail_expectation.json")
    M = t["max_len"]
    for B in t["block_sizes"]:
        # exact enumeration over 1..512 equals the closed form (B - 1) / 2
        assert acc.mean_tail_waste_exact(B, M) == acc.expected_tail_waste(B) == Fraction(B - 1, 2)
        # bound W_tail <= N (B - 1), reached when every length is 1 mod B
        lengths = list(range(1, M + 1))
        assert acc.waste_table(lengths, B)[3] <= acc.tail_waste_bound(len(lengths), B)
        worst = [1 + k * B for k in range(8)]
        assert acc.waste_table(worst, B)[3] == acc.tail_waste_bound(len(worst), B)
    assert acc.mean_fixed_waste_exact(M) == Fraction(t["fixed_reservation_mean_waste"]).limit_denominator()
    # tail waste of a non-empty request lies in [0, B - 1]
    for B in (4, 16, 64):
        assert all(0 <= acc.tail_waste(n, B) <= B - 1 for n in range(1, 4 * B))


# -- pool capacity ------------------------------------------------------------
def test_capacity_24gib():
    c = golden("capacity.json")["pool_24gib"]
    nb = acc.pool_blocks(c["pool_gib"] * GiB, c["bytes_per_token"], c["block_size"])
    assert nb == c["blocks"]
    assert acc.blocks_needed(c["request_tokens"], c["block_size"]) == c["blocks_per_request"]
    fit, left = acc.requests_that_fit(nb, c["request_tokens"], c["block_size"])
    assert (fit, left) == (c["requests"], c["blocks_left"])
    assert fit * c["blocks_per_request"] == c["blocks_used"]
    assert c["blocks_per_request"] - left == c["next_request_short_by"]


def test_capacity_24gib_allocator():
    """The allocator itself admits 47 requests of 4112 tokens and fails the 48th cleanly."""
    c = golden("capacity.json")["pool_24gib"]
    a = RefAllocator(c["blocks"], c["block_size"])
    for i in range(c["requests"]):
        assert a.add_seq(i, c["request_tokens"]) == OK
    st = a.stats()
    assert st["free"] == c["blocks_left"] and st["active"] == c["blocks_used"]
    before = (list(a.free), list(a.ref), {k: a.table(k) for k in a.seqs})
    assert a.add_seq(c["requests"], c["request_tokens"]) == NO_BLOCKS
    assert (list(a.free), list(a.ref), {k: a.table(k) for k in a.seqs}) == before
    assert a.check()


def test_capacity_8gib():
    c = golden("capacity.json")["pool_8gib"]
    block_bytes = c["bytes_per_token"] * c["block_size"]
    assert block_bytes == c["block_kib"] * KiB
    nb = acc.pool_blocks(c["pool_gib"] * GiB, c["bytes_per_token"], c["block_size"])
    assert nb == c["blocks"]
    assert (c["pool_gib"] * GiB - nb * block_bytes) == c["unallocated_kib"] * KiB
    fit, left = acc.requests_that_fit(nb, c["request_tokens"], c["block_size"])
    assert acc.blocks_needed(c["request_tokens"], c["block_size"]) == c["blocks_per_request"]
    assert (fit, left) == (c["requests"], c["blocks_left"])
    a = RefAllocator(nb, c["block_size"])
    for i in range(fit):
        assert a.add_seq(i, c["request_tokens"]) == OK
    assert a.stats()["free"] == c["blocks_left"]
    assert a.add_seq(fit, c["request_tokens"]) == NO_BLOCKS
    assert a.check()


def test_swap_time():
    s = golden("swap.json")
    one = acc.swap_seconds(s["mib"] * MiB, s["link_gib_per_s"] * GiB) * 1000
    assert round(one, s["printed_decimals"]) == s["one_way_ms"]
    assert round(2 * one, s["printed_decimals"]) == s["round_trip_ms"]


# -- block table, address mapping --------------------------------------------
def test_address_mapping_token_6():
    m = golden("address_mapping.json")
    lb, off = kvops.logical_address(m["token"], m["block_size"])
    assert (lb, off) == (m["logical_block"], m["offset"])
    assert m["table"][lb] == m["physical_block"]
    assert kvops.slot_of(m["table"], m["token"], m["block_size"]) == m["physical_block"] * m["block_size"] + m["offset"]


def test_address_mapping_through_pool():
    """The token written through the table is found at [physical, offset] of the pool."""
    import numpy as np

    m = golden("address_mapping.json")
    B, table = m["block_size"], m["table"]
    pool = kvops.new_pool(8, B, 2, 4, np.float32)
    hist = np.arange(10 * 2 * 4, dtype=np.float32).reshape(10, 2, 4)
    kvops.scatter_history(pool, table, hist)
    assert np.array_equal(pool[m["physical_block"], m["offset"]], hist[m["token"]])
    assert np.array_equal(kvops.gather_history(pool, table, 10), hist)


# -- allocator walkthroughs ---------------------------------------------------
def _p(name):
    return int(name[1:])


def test_cow_walkthrough():
    """B = 4; A and B share the partial tail P2; 5 free blocks (a 6-block pool)."""
    w = golden("cow.json")["walkthrough"]
    B = w["block_size"]
    # P2 is taken first (the shared tail), then P3 is the next free block.
    a = RefAllocator(6, B, free_order=[2, 3, 0, 1, 4, 5])
    assert a.add_seq(0, 3) == OK           # request A: 3 tokens in P2
    assert a.fork(0, 1) == OK              # request B shares P2
    assert a.table(0) == [_p(w["shared_tail"])]
    assert a.ref[_p(w["shared_tail"])] == w["shared_refcount_before"]
    assert a.stats()["free"] == w["free_before"]
    s1, s2, s3 = w["steps"]
    st, per, copies = a.append([0])        # A writes: COW into P3
    assert st == OK and per == [OK]
    assert copies == [(_p(w["shared_tail"]), _p(s1["new_block"]), 3)]
    assert a.table(0) == [_p(s1["new_block"])] and a.table(1) == [_p(w["shared_tail"])]
    for blk, r in s1["refcounts"].items():
        assert a.ref[_p(blk)] == r
    assert a.stats()["free"] == s1["free"] and a.check()
    assert a.free_seq(0) == OK             # A finishes
    for blk, r in s2["refcounts"].items():
        assert a.ref[_p(blk)] == r
    assert a.stats()["free"] == s2["free"] and a.check()
    assert a.free_seq(1) == OK             # B finishes
    for blk, r in s3["refcounts"].items():
        assert a.ref[_p(blk)] == r
    assert a.stats()["free"] == s3["free"] == 6 and a.check()


def test_cow_content_isolation():
    """Shared tail P3 holds a,b,c; B gets P8 = copy(a,b,c); A writes X in P3, B writes Y in P8."""
    import numpy as np

    c = golden("cow.json")["content_isolation"]
    B = c["block_size"]
    order = [3, 8] + [b for b in range(10) if b not in (3, 8)]
    a = RefAllocator(10, B, free_order=order)
    tok = {"a": 1.0, "b": 2.0, "c": 3.0, "X": 24.0, "Y": 25.0}
    pool = kvops.new_pool(10, B, 1, 1, np.float32, fill=np.nan)
    assert a.add_seq(0, 3) == OK           # A holds a, b, c in P3
    kvops.scatter_history(pool, a.table(0), np.array([[[tok[t]]] for t in c["tail_tokens"]], np.float32))
    assert a.fork(0, 1) == OK
    st, per, copies = a.append([1, 0])     # B first: it sees refcount 2 and copies
    assert st == OK
    assert copies == [(_p(c["shared_tail"]), _p(c["B_new_block"]), len(c["tail_tokens"]))]
    kvops.block_copy([pool], copies)
    slots = kvops.slot_mapping([a.table(1), a.table(0)], [0, 1], [a.length(1) - 1, a.length(0) - 1], B)
    kvops.append(pool, slots, np.array([[[tok[c["B_writes"]]]], [[tok[c["A_writes"]]]]], np.float32))
    for blk, toks in c["after"].items():
        assert pool[_p(blk), :, 0, 0].tolist() == [tok[t] for t in toks]
    assert a.table(0) == [_p(c["shared_tail"])] and a.table(1) == [_p(c["B_new_block"])]
    assert a.check()


def test_append_across_block():
    c = golden("cow.json")["append_across_block"]
    B = c["block_size"]
    a = RefAllocator(8, B, free_order=[5, 2, 0, 1, 3, 4, 6, 7])
    assert a.add_seq(0, c["tokens_before"]) == OK
    assert a.table(0) == [_p(p) for p in c["table_before"]]
    st, per, copies = a.append([0])
    assert st == OK and copies == []
    assert a.table(0) == [_p(p) for p in c["table_after"]]
    lb, off = kvops.logical_address(c["new_token"], B)
    assert a.table(0)[lb] == _p(c["new_block"]) and off == 0
    assert a.check()


def test_admission_three_of_four():
    c = golden("cow.json")["admission"]
    B = 4
    n_req = len(c["requests"])
    a = RefAllocator(n_req + c["free"], B)
    for i in range(n_req):
        assert a.add_seq(i, B) == OK        # full tails: each needs one new block
    assert a.stats()["free"] == c["free"]
    before_last = (a.table(n_req - 1), a.length(n_req - 1))
    st, per, copies = a.append(list(range(n_req)))
    assert st == NO_BLOCKS
    assert per.count(OK) == c["run"] and per.count(NO_BLOCKS) == c["wait"]
    assert per == [OK] * c["run"] + [NO_BLOCKS] * c["wait"]
    assert (a.table(n_req - 1), a.length(n_req - 1)) == before_last
    assert a.check()


def test_teaching_log_conservation():
    c = golden("capacity.json")["teaching_log"]
    B = 4
    a = RefAllocator(c["pool"], B, enable_cache=True)
    # 100 requests of 10 full blocks each use the whole pool
    for i in range(100):
        assert a.add_seq(i, 10 * B) == OK
    # 30 of them finish: their full blocks stay cached (evictable), not free
    for i in range(30):
        assert a.free_seq(i) == OK
    st = a.stats()
    assert (st["active"], st["cached"], st["free"]) == (c["active"], c["cached"], c["free"])
    assert st["active"] + st["cached"] + st["free"] == c["pool"]
    assert a.available() == c["cached"]
    assert a.add_seq(1000, c["request_blocks"] * B) == NO_BLOCKS
    assert c["request_blocks"] - a.available() == c["short_by"]
    # a request that fits evicts cached blocks oldest first
    first_cached = a.cached[0]
    assert a.add_seq(1001, 2 * B) == OK and a.table(1001)[0] == first_cached
    assert a.check()


def test_invalid_ops_change_nothing():
    a = RefAllocator(8, 4)
    assert a.add_seq(0, 5) == OK
    snap = (list(a.free), list(a.ref), a.table(0), a.length(0))
    assert a.add_seq(0, 1) == INVALID
    assert a.fork(7, 8) == INVALID
    assert a.fork(0, 0) == INVALID
    assert a.append([0, 0])[0] == INVALID
    assert a.append([0, 99])[0] == INVALID
    assert a.free_seq(42) == INVALID
    assert (list(a.free), list(a.ref), a.table(0), a.length(0)) == snap
    assert a.check()


def test_leak_is_detected():
    """A release that skips the refcount decrement leaves the recount wrong."""
    class LeakyAllocator(RefAllocator):
        def free_seq(self, seq_id):
            if seq_id not in self.seqs:
                return INVALID
            self.seqs.pop(seq_id)   # planted mistake: references never dropped
            return OK

    a = LeakyAllocator(16, 4)
    for i in range(4):
        assert a.add_seq(i, 8) == OK
    assert a.check()
    assert a.free_seq(0) == OK
    assert not a.check()
    # repeated leaks drain the pool: admission fails although no request is live
    b = LeakyAllocator(16, 4)
    for i in range(8):
        assert b.add_seq(i, 8) == OK
        assert b.free_seq(i) == OK
    assert b.add_seq(100, 4) == NO_BLOCKS and len(b.seqs) == 0


def test_cow_allocation_failure_keeps_mapping():
    a = RefAllocator(2, 4, free_order=[0, 1])
    assert a.add_seq(0, 3) == OK
    assert a.fork(0, 1) == OK
    assert a.add_seq(2, 4) == OK             # last free block gone
    snap = (a.table(0), a.table(1), list(a.ref), a.length(0))
    st, per, copies = a.append([0])
    assert st == NO_BLOCKS and per == [NO_BLOCKS] and copies == []
    assert (a.table(0), a.table(1), list(a.ref), a.length(0)) == snap
    assert a.check()


def test_random_ops_keep_invariant():
    import random

    rnd = random.Random(7)
    for cache in (False, True):
        a = RefAllocator(64, 4, free_order=rnd.sample(range(64), 64), enable_cache=cache)
        live = []
        nxt = 0
        for _ in range(2000):
            op = rnd.random()
            if op < 0.25 or not live:
                if a.add_seq(nxt, rnd.randint(0, 12)) == OK:
                    live.append(nxt)
                nxt += 1
            elif op < 0.4:
                if a.fork(rnd.choice(live), nxt) == OK:
                    live.append(nxt)
                nxt += 1
            elif op < 0.85:
                ids = rnd.sample(live, rnd.randint(1, len(live)))
                a.append(ids)
            else:
                sid = live.pop(rnd.randrange(len(live)))
                assert a.free_seq(sid) == OK
            assert a.check()
        for sid in live:
            a.free_seq(sid)
        st = a.stats()
        assert st["active"] == 0 and st["free"] + st["cached"] == 64
