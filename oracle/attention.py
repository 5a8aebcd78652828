"""Decode attention in binary64 (oracle; test infrastructure only).

What the method computes has a plain definition: one query token per request
attends over that request's whole history, exactly as dense attention over the
contiguous K/V would ([P2] "PagedAttention：让 KV cache 按需生长", section
"分页以后，attention 仍然按完整历史归一化"; [P3] "内存预算约束下的语言模型服务：注意力、分页与调度",
section "6. 精确注意力仍有数值契约").  So the oracle is that definition:

    s_t = scale * <q_h, K_t[g(h)]>,   p = softmax(s),   out_h = sum_t p_t V_t[g(h)]

with grouped-query heads g(h) = h // (H_q / H_kv) (query heads that share a KV
head are adjacent; the pages leave the grouping open and this is the plainest
reading).  The softmax subtracts max(s) before exponentiating; that is the same
function and keeps |s| ~ 1e3 finite.  An empty history (length 0) gives 0.

Two further functions restate the paged algorithm itself so it can be checked
against the definition:

* ``paged_online_decode`` walks the logical blocks in order, looks up the
  physical block, masks slots at or past the length to -inf and applies the
  online-softmax recurrence of [P3] equation (4): m' = max(m, max_j s_j),
  l' = e^{m-m'} l + sum_j e^{s_j-m'}, with the value accumulator rescaled by the
  same factor.  Masked slots never enter any sum (they may hold NaN).
* ``merge_states`` combines partial (m, l, o) states of disjoint token ranges;
  [P2]'s third exercise ("逻辑顺序没错，为什么 attention 输出还是错？") states
  that these states merge where per-block softmax outputs cannot be averaged.
"""
from __future__ import annotations

from typing import Iterable, List, Sequence, Tuple

import numpy as np


def widen(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) or float32/float64 values -> exact float64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def dense_decode(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, scale: float) -> np.ndarray:
    """Dense attention of one request.

    q: [H_q, d]; k_hist, v_hist: [n, H_kv, d] (any dtype ``widen`` accepts).
    Returns float64 [H_q, d].
    """
    q = widen(q)
    K = widen(k_hist)
    V = widen(v_hist)
    H_q, d = q.shape
    n, H_kv = K.shape[0], K.shape[1]
    if H_q % H_kv:
        raise ValueError("H_q must be a multiple of H_kv")
    G = H_q // H_kv
    out = np.zeros((H_q, d), dtype=np.float64)
    if n == 0:
        return out
    for h in range(H_q):
        g = h // G
        s = float(scale) * (K[:, g, :] @ q[h])
        e = np.exp(s - s.max())
        p = e / e.sum()
        out[h] = p @ V[:, g, :]
    return out


def dense_decode_head(q_h: np.ndarray, k_head: np.ndarray, v_head: np.ndarray, scale: float) -> np.ndarray:
    """Dense attention of one query head over one KV head: q_h [d], k/v [n, d]."""
    qh = widen(q_h)
    K = widen(k_head)
    V = widen(v_head)
    if K.shape[0] == 0:
        return np.zeros(qh.shape[0], dtype=np.float64)
    s = float(scale) * (K @ qh)
    e = np.exp(s - s.max())
    return (e / e.sum()) @ V


def paged_decode(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray,
                 tables: Sequence[Sequence[int]], seq_lens: Sequence[int], scale: float) -> np.ndarray:
    """Reference for a batch: gather each history through its table, then dense.

    q: [S, H_q, d]; pools [N_blk, B, H_kv, d]; returns float64 [S, H_q, d].
    """
    from .kvops import gather_history

    S = q.shape[0]
    out = np.zeros(q.shape, dtype=np.float64)
    for s in range(S):
        n = int(seq_lens[s])
        kh = gather_history(k_pool, tables[s], n)
        vh = gather_history(v_pool, tables[s], n)
        out[s] = dense_decode(q[s], kh, vh, scale)
    return out


def multi_query(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, scale: float) -> np.ndarray:
    """T query tokens of one request at the last T positions of its history.

    The staged positions of speculative decoding ([P1] "PagedAttention 与在线推理：KV
    分页、共享及调度的联合分析", section 5) are verified by running every staged
    token's query at once; each token attends causally, i.e. only up to its own
    position, with the attention of [P3] section 6.  q: [T, H_q, d];
    k_hist, v_hist: [n, H_kv, d] holding all n tokens including the T new ones.
    Token i sits at position p = n - T + i and is dense decode over the first
    p + 1 tokens; p < 0 (fewer than T - i tokens) attends nothing and gives 0.
    Returns float64 [T, H_q, d].
    """
    T = q.shape[0]
    n = k_hist.shape[0]
    out = np.zeros((T,) + q.shape[1:], dtype=np.float64)
    for i in range(T):
        p = n - T + i
        if p >= 0:
            out[i] = dense_decode(q[i], k_hist[:p + 1], v_hist[:p + 1], scale)
    return out


State = Tuple[np.ndarray, np.ndarray, np.ndarray]  # m [H], l [H], o [H, d]


def empty_state(H: int, d: int) -> State:
    return (np.full(H, -np.inf), np.zeros(H), np.zeros((H, d)))


def online_update(state: State, s: np.ndarray, v: np.ndarray) -> State:
    """Equation (4) of P3 for one block of scores.

    s: [H, j] scores of the block's valid slots; v: [H, j, d] their values.
    """
    m, l, o = state
    if s.shape[1] == 0:
        return state
    m_new = np.maximum(m, s.max(axis=1))
    alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
    e = np.exp(s - m_new[:, None])
    l_new = alpha * l + e.sum(axis=1)
    o_new = alpha[:, None] * o + np.einsum("hj,hjd->hd", e, v)
    return (m_new, l_new, o_new)


def finish(state: State) -> np.ndarray:
    """o / l, and 0 where nothing was attended (l = 0)."""
    m, l, o = state
    out = np.zeros_like(o)
    nz = l > 0
    out[nz] = o[nz] / l[nz][:, None]
    return out


def merge_states(states: Iterable[State]) -> State:
    """Combine partial states of disjoint token ranges into one."""
    states = list(states)
    H, d = states[0][2].shape
    M = np.full(H, -np.inf)
    for m, _, _ in states:
        M = np.maximum(M, m)
    l_tot = np.zeros(H)
    o_tot = np.zeros((H, d))
    for m, l, o in states:
        w = np.where(np.isneginf(m), 0.0, np.exp(m - np.where(np.isneginf(M), 0.0, M)))
        l_tot += w * l
        o_tot += w[:, None] * o
    return (M, l_tot, o_tot)


def paged_online_decode(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray,
                        table: Sequence[int], length: int, scale: float) -> np.ndarray:
    """The paged loop for one request, in the order the page gives its steps.

    For each logical block: physical = table[block]; load that block's K and V
    tile; valid = block * B + arange(B) < length; scores = (q K^T) * scale with
    invalid slots at -inf; online-softmax update.  Returns float64 [H_q, d].
    """
    qf = widen(q)
    H_q, d = qf.shape
    B, H_kv = k_pool.shape[1], k_pool.shape[2]
    G = H_q // H_kv
    nblk = -(-int(length) // B)
    state = empty_state(H_q, d)
    for lb in range(nblk):
        phys = int(table[lb])
        K_tile = widen(k_pool[phys])          # [B, H_kv, d]
        V_tile = widen(v_pool[phys])
        valid = lb * B + np.arange(B) < length
        kv_head = np.arange(H_q) // G
        scores = np.full((H_q, B), -np.inf)
        for h in range(H_q):
            kh = K_tile[valid, kv_head[h], :]
            scores[h, valid] = float(scale) * (kh @ qf[h])
        sv = scores[:, valid]
        vv = np.stack([V_tile[valid, kv_head[h], :] for h in range(H_q)], axis=0)
        state = online_update(state, sv, vv)
    return finish(state)


def online_decode_blocks(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, scale: float,
                         block: int) -> np.ndarray:
    """Online recurrence over a contiguous history cut into blocks of ``block``."""
    qf = widen(q)
    K = widen(k_hist)
    V = widen(v_hist)
    H_q, d = qf.shape
    n, H_kv = K.shape[0], K.shape[1]
    G = H_q // H_kv
    kv_head = np.arange(H_q) // G
    state = empty_state(H_q, d)
    for t0 in range(0, n, block):
        t1 = min(n, t0 + block)
        s = np.stack([float(scale) * (K[t0:t1, kv_head[h], :] @ qf[h]) for h in range(H_q)])
        v = np.stack([V[t0:t1, kv_head[h], :] for h in range(H_q)])
        state = online_update(state, s, v)
    return finish(state)


def split_states(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, scale: float,
                 cuts: Sequence[int]) -> List[State]:
    """Partial states of the token ranges [cuts[i], cuts[i+1]) (for merge checks)."""
    qf = widen(q)
    K = widen(k_hist)
    V = widen(v_hist)
    H_q, d = qf.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    kv_head = np.arange(H_q) // G
    out = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        st = empty_state(H_q, d)
        if b > a:
            s = np.stack([float(scale) * (K[a:b, kv_head[h], :] @ qf[h]) for h in range(H_q)])
            v = np.stack([V[a:b, kv_head[h], :] for h in range(H_q)])
            st = online_update(st, s, v)
        out.append(st)
    return out
