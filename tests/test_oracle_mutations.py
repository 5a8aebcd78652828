"""Planted mistakes in the oracle must fail at least one pin.

Each mutant below is a plausible slip (a wrong index, a dropped term, a
transposed operand, a wrong queue end).  It is planted in a copy of the oracle
function on the CPU, and the pins of tests/test_oracle_*.py that should catch
it are re-run against it.  The unmodified oracle passes the same checks.
"""
import numpy as np
import pytest

from oracle import attention as att
from oracle import kvops
from oracle.allocator import OK, RefAllocator
from tests import test_oracle_attention as TA
from tests import test_oracle_pins as TP


# -- attention mutants --------------------------------------------------------
def _dense_wrong_gqa(q, k_hist, v_hist, scale):
    q, K, V = att.widen(q), att.widen(k_hist), att.widen(v_hist)
    H_q, d = q.shape
    H_kv = K.shape[1]
    out = np.zeros((H_q, d))
    if K.shape[0] == 0:
        return out
    for h in range(H_q):
        g = h % H_kv                      # interleaved instead of grouped heads
        s = scale * (K[:, g] @ q[h])
        e = np.exp(s - s.max())
        out[h] = (e / e.sum()) @ V[:, g]
    return out


def _dense_no_scale(q, k_hist, v_hist, scale):
    return att.__dict__["_orig_dense"](q, k_hist, v_hist, 1.0)


def _dense_keys_as_values(q, k_hist, v_hist, scale):
    return att.__dict__["_orig_dense"](q, k_hist, k_hist, scale)


def _dense_no_max_shift(q, k_hist, v_hist, scale):
    q, K, V = att.widen(q), att.widen(k_hist), att.widen(v_hist)
    H_q, d = q.shape
    G = H_q // K.shape[1]
    out = np.zeros((H_q, d))
    if K.shape[0] == 0:
        return out
    with np.errstate(over="ignore", invalid="ignore"):
        for h in range(H_q):
            e = np.exp(scale * (K[:, h // G] @ q[h]))
            out[h] = (e / e.sum()) @ V[:, h // G]
    return out


def _gather_off_by_one(pool, table, length):
    B = pool.shape[1]
    if length == 0:
        return pool[:0, 0]
    return np.stack([pool[int(table[(t + 1) // B if (t + 1) // B < len(table) else 0]), t % B]
                     for t in range(length)])


def _online_no_rescale(state, s, v):
    m, l, o = state
    if s.shape[1] == 0:
        return state
    m_new = np.maximum(m, s.max(axis=1))
    e = np.exp(s - m_new[:, None])
    return (m_new, l + e.sum(axis=1), o + np.einsum("hj,hjd->hd", e, v))   # alpha dropped


ATTN_PINS = [
    lambda: [TA.test_dense_matches_torch_sdpa(*c) for c in [(5, 8, 2, 16), (17, 16, 4, 32)]],
    lambda: TA.test_length_one_returns_v0(),
    lambda: TA.test_permuted_blocks_and_poisoned_tails_match_dense(4),
    lambda: TA.test_online_recurrence_matches_dense_witness(),
    lambda: TA.test_extreme_logits_stay_finite(1000.0),
]


def _any_pin_fails(pins):
    for pin in pins:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            return True
    return False


def test_unmutated_oracle_passes_attention_pins():
    assert not _any_pin_fails(ATTN_PINS)


@pytest.mark.parametrize("mutant", [_dense_wrong_gqa, _dense_no_scale, _dense_keys_as_values,
                                    _dense_no_max_shift])
def test_dense_mutants_are_caught(monkeypatch, mutant):
    monkeypatch.setitem(att.__dict__, "_orig_dense", att.dense_decode)
    monkeypatch.setattr(att, "dense_decode", mutant)
    assert _any_pin_fails(ATTN_PINS)


def test_gather_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(kvops, "gather_history", _gather_off_by_one)
    assert _any_pin_fails(ATTN_PINS)


def test_online_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(att, "online_update", _online_no_rescale)
    assert _any_pin_fails(ATTN_PINS)


# -- allocator mutants --------------------------------------------------------
class _Lifo(RefAllocator):
    def _take(self):
        b = self.free.pop()                 # takes from the wrong end
        self.ref[b] = 1
        self.counters["allocs"] += 1
        return b


class _NoTailDecrement(RefAllocator):
    def append(self, seq_ids):
        B = self.block_size
        statuses, copies = [], []
        for sid in seq_ids:
            s = self.seqs[sid]
            n = s.length
            if n % B == 0:
                s.table.append(self._take())
            elif self.ref[s.table[-1]] > 1:
                new = self._take()
                copies.append((s.table[-1], new, n % B))
                s.table[-1] = new                # refcount of the old tail never drops
            s.length = n + 1
            statuses.append(OK)
        return OK, statuses, copies


class _CopyWholeLength(RefAllocator):
    def append(self, seq_ids):
        st, per, copies = super().append(seq_ids)
        return st, per, [(a, b, self.seqs[seq_ids[0]].length - 1) for a, b, _ in copies]


ALLOC_PINS = [TP.test_cow_walkthrough, TP.test_cow_content_isolation, TP.test_append_across_block,
              TP.test_admission_three_of_four, TP.test_capacity_24gib_allocator]


def test_unmutated_allocator_passes_pins():
    assert not _any_pin_fails(ALLOC_PINS)


@pytest.mark.parametrize("mutant", [_Lifo, _NoTailDecrement])
def test_allocator_mutants_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(TP, "RefAllocator", mutant)
    assert _any_pin_fails(ALLOC_PINS)


def test_copy_length_mutant_is_caught():
    """A COW that copies the whole length instead of n mod B: the tail past a full block."""
    for cls, expect_ok in ((RefAllocator, True), (_CopyWholeLength, False)):
        a = cls(8, 4)
        assert a.add_seq(0, 7) == OK            # one full block + 3 tokens in the tail
        assert a.fork(0, 1) == OK
        st, per, copies = a.append([0])
        good = copies == [(a.table(1)[1], a.table(0)[1], 3)] and a.table(0)[0] == a.table(1)[0] \
            and a.ref[a.table(0)[0]] == 2
        assert good == expect_ok


# -- multi-token query mutant -------------------------------------------------
def _multi_query_off_by_one(q, k_hist, v_hist, scale):
    T, n = q.shape[0], k_hist.shape[0]
    out = np.zeros((T,) + q.shape[1:])
    for i in range(T):
        p = n - T + i
        if p >= 0:       # sees one token past its own position
            out[i] = att.dense_decode(q[i], k_hist[:p + 2], v_hist[:p + 2], scale)
    return out


MQ_PINS = [lambda: TA.test_multi_query_matches_torch_causal_sdpa(9, 3, 8, 2, 16),
           TA.test_multi_query_special_cases]


def test_unmutated_multi_query_passes_pins():
    assert not _any_pin_fails(MQ_PINS)


def test_multi_query_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(att, "multi_query", _multi_query_off_by_one)
    assert _any_pin_fails(MQ_PINS)


# -- per-head checker and bf16 decoder mutants ---------------------------------
def _head_no_max_shift(q_h, k_head, v_head, scale):
    qh, K, V = att.widen(q_h), att.widen(k_head), att.widen(v_head)
    if K.shape[0] == 0:
        return np.zeros(qh.shape[0])
    e = np.exp(float(scale) * (K @ qh))     # overflows at |s| ~ 1e3
    return (e / e.sum()) @ V


def _head_scale_squared(q_h, k_head, v_head, scale):
    return att.__dict__["_orig_head"](q_h, k_head, v_head, float(scale) ** 2)


def _widen_shift_15(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


HEAD_PINS = [lambda: TA.test_dense_decode_head_matches_sdpa(64, 32, 4, 128, "bf16", 1000.0),
             lambda: TA.test_dense_decode_head_matches_sdpa(5, 8, 2, 16, "f32", 1.0),
             TA.test_dense_decode_head_special_cases]
WIDEN_PINS = [TA.test_widen_matches_torch_bfloat16]


def test_unmutated_head_and_widen_pass_pins():
    assert not _any_pin_fails(HEAD_PINS)
    assert not _any_pin_fails(WIDEN_PINS)


@pytest.mark.parametrize("mutant", [_head_no_max_shift, _head_scale_squared])
def test_head_mutants_are_caught(monkeypatch, mutant):
    monkeypatch.setitem(att.__dict__, "_orig_head", att.dense_decode_head)
    monkeypatch.setattr(att, "dense_decode_head", mutant)
    assert _any_pin_fails(HEAD_PINS)


def test_widen_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(att, "widen", _widen_shift_15)
    assert _any_pin_fails(WIDEN_PINS)
