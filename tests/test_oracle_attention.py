"""The oracle's attention against things other than itself.

Pins:
* a library routine: torch's scaled_dot_product_attention in float64 on the
  CPU, with grouped-query heads expanded by repeat_interleave (query head h
  reads KV head h // G), on contiguous histories;
* closed-form special cases: length 1 gives v_0, equal keys give the mean of
  V, one dominant logit gives that token's v, length 0 gives 0;
* invariances the pages ask for: randomly permuted physical block ids, slots
  past the length poisoned with NaN;
* the paged online recurrence and the merge of split states against the dense
  definition in binary64 (P3's executed check reports 2.22e-16 over 8 cases);
* extreme logits (|s| ~ 1e3) stay finite and agree.
"""
import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import kvops
from oracle.allocator import OK, RefAllocator
from tests.conftest import golden
from workloads import normal_bf16_bits, normal_f32, rng


def _sdpa_f64(q, K, V, scale):
    """q [H_q, d], K/V [n, H_kv, d] float64 -> [H_q, d] via torch SDPA."""
    H_q = q.shape[0]
    H_kv = K.shape[1]
    G = H_q // H_kv
    qt = torch.from_numpy(q)[:, None, :]                     # [H_q, 1, d]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, dim=0)  # [H_q, n, d]
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, dim=0)
    out = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], scale=scale)
    return out[0, :, 0, :].numpy()


@pytest.mark.parametrize("n,H_q,H_kv,d", [(1, 4, 1, 8), (5, 8, 2, 16), (37, 8, 2, 64), (200, 32, 8, 128),
                                          (17, 16, 4, 32), (64, 32, 4, 128)])
def test_dense_matches_torch_sdpa(n, H_q, H_kv, d):
    g = rng(100 + n)
    q = normal_f32(g, (H_q, d)).astype(np.float64)
    K = normal_f32(g, (n, H_kv, d)).astype(np.float64)
    V = normal_f32(g, (n, H_kv, d)).astype(np.float64)
    scale = 1.0 / np.sqrt(d)
    ref = _sdpa_f64(q, K, V, scale)
    out = att.dense_decode(q, K, V, scale)
    assert np.max(np.abs(out - ref)) < 1e-13


def test_length_one_returns_v0():
    g = rng(1)
    q = normal_bf16_bits(g, (8, 64))
    K = normal_bf16_bits(g, (1, 2, 64))
    V = normal_bf16_bits(g, (1, 2, 64))
    out = att.dense_decode(q, K, V, 0.125)
    Vf = att.widen(V)
    for h in range(8):
        assert np.array_equal(out[h], Vf[0, h // 4])


def test_length_zero_is_zero():
    out = att.dense_decode(np.ones((4, 8), np.float32), np.zeros((0, 2, 8), np.float32),
                           np.zeros((0, 2, 8), np.float32), 0.5)
    assert np.array_equal(out, np.zeros((4, 8)))


def test_equal_keys_give_mean_of_values():
    g = rng(2)
    n, H_kv, d = 50, 2, 16
    q = normal_f32(g, (4, d))
    K = np.repeat(normal_f32(g, (1, H_kv, d)), n, axis=0)
    V = normal_f32(g, (n, H_kv, d))
    out = att.dense_decode(q, K, V, 0.25)
    for h in range(4):
        np.testing.assert_allclose(out[h], V.astype(np.float64)[:, h // 2].mean(axis=0), rtol=0, atol=1e-14)


def test_dominant_logit_selects_value():
    g = rng(3)
    n, d = 40, 32
    K = normal_f32(g, (n, 1, d))
    V = normal_f32(g, (n, 1, d))
    star = 17
    q = (K[star, 0] * 1000.0)[None, :]
    out = att.dense_decode(q, K, V, 1.0)
    np.testing.assert_allclose(out[0], V[star, 0].astype(np.float64), rtol=0, atol=1e-12)


def _paged_setup(lengths, B, H_kv, d, seed, dtype="f32", poison=True):
    g = rng(seed)
    nb = sum(-(-n // B) for n in lengths) + 3
    perm = g.permutation(nb)
    a = RefAllocator(nb, B, free_order=perm)
    for i, n in enumerate(lengths):
        assert a.add_seq(i, n) == OK
    if dtype == "f32":
        fill = np.nan if poison else 0.0
        kp = kvops.new_pool(nb, B, H_kv, d, np.float32, fill)
        vp = kvops.new_pool(nb, B, H_kv, d, np.float32, fill)
        hk = [normal_f32(g, (n, H_kv, d)) for n in lengths]
        hv = [normal_f32(g, (n, H_kv, d)) for n in lengths]
    else:
        fill = 0x7FC0 if poison else 0
        kp = kvops.new_pool(nb, B, H_kv, d, np.uint16, fill)
        vp = kvops.new_pool(nb, B, H_kv, d, np.uint16, fill)
        hk = [normal_bf16_bits(g, (n, H_kv, d)) for n in lengths]
        hv = [normal_bf16_bits(g, (n, H_kv, d)) for n in lengths]
    for i in range(len(lengths)):
        kvops.scatter_history(kp, a.table(i), hk[i])
        kvops.scatter_history(vp, a.table(i), hv[i])
    tables = [a.table(i) for i in range(len(lengths))]
    return kp, vp, tables, hk, hv


@pytest.mark.parametrize("B", [4, 16, 64])
def test_permuted_blocks_and_poisoned_tails_match_dense(B):
    """Random physical ids, NaN in every unwritten slot, lengths 0/1/B/B+1 and more."""
    lengths = [0, 1, B, B + 1, 37, 91, 2 * B - 1]
    H_q, H_kv, d = 8, 2, 16
    kp, vp, tables, hk, hv = _paged_setup(lengths, B, H_kv, d, seed=B)
    g = rng(500 + B)
    q = normal_f32(g, (len(lengths), H_q, d))
    scale = 1 / 4
    out = att.paged_decode(q, kp, vp, tables, lengths, scale)
    assert np.all(np.isfinite(out))
    for i, n in enumerate(lengths):
        ref = _sdpa_f64(q[i].astype(np.float64), hk[i].astype(np.float64), hv[i].astype(np.float64), scale) \
            if n > 0 else np.zeros((H_q, d))
        assert np.max(np.abs(out[i] - ref)) < 1e-13
        online = att.paged_online_decode(q[i], kp, vp, tables[i], n, scale)
        assert np.all(np.isfinite(online))
        assert np.max(np.abs(online - out[i])) < 1e-14


def test_online_recurrence_matches_dense_witness():
    """P3's executed check: binary64 online softmax vs dense over 8 cases and several block sizes."""
    w = golden("witness.json")
    worst = 0.0
    cases = 0
    for case in range(w["attention_cases"]):
        g = rng(900 + case)
        n = int(g.integers(1, 300))
        q = normal_f32(g, (4, 32)).astype(np.float64)
        K = normal_f32(g, (n, 2, 32)).astype(np.float64)
        V = normal_f32(g, (n, 2, 32)).astype(np.float64)
        dense = att.dense_decode(q, K, V, 1 / np.sqrt(32))
        for blk in (1, 4, 16, 64):
            online = att.online_decode_blocks(q, K, V, 1 / np.sqrt(32), blk)
            worst = max(worst, float(np.max(np.abs(online - dense))))
        cases += 1
    assert cases == w["attention_cases"]
    # same order of magnitude as the printed 2.22e-16: a few ulps of |out| <= 1
    assert worst <= 8 * w["largest_absolute_error"]


def test_merge_of_split_states_matches_dense():
    g = rng(11)
    n = 777
    q = normal_f32(g, (8, 64))
    K = normal_f32(g, (n, 2, 64))
    V = normal_f32(g, (n, 2, 64))
    dense = att.dense_decode(q, K, V, 0.125)
    for cuts in ([0, n], [0, 1, n], [0, 100, 100, 400, n], list(range(0, n, 64)) + [n]):
        merged = att.finish(att.merge_states(att.split_states(q, K, V, 0.125, cuts)))
        assert np.max(np.abs(merged - dense)) < 1e-14


def test_equal_weight_average_of_blocks_is_wrong():
    """P2's third exercise: averaging per-block softmax outputs loses the normalisation."""
    g = rng(12)
    n = 40
    q = normal_f32(g, (1, 16), 3.0)
    K = normal_f32(g, (n, 1, 16))
    V = normal_f32(g, (n, 1, 16))
    dense = att.dense_decode(q, K, V, 0.25)
    per_block = [att.dense_decode(q, K[a:a + 16], V[a:a + 16], 0.25) for a in range(0, n, 16)]
    assert np.max(np.abs(np.mean(per_block, axis=0) - dense)) > 1e-3


@pytest.mark.parametrize("qscale", [30.0, 1000.0])
def test_extreme_logits_stay_finite(qscale):
    g = rng(13)
    n, d = 300, 128
    q = normal_bf16_bits(g, (32, d), qscale)
    K = normal_bf16_bits(g, (n, 8, d))
    V = normal_bf16_bits(g, (n, 8, d))
    scale = 1 / np.sqrt(d)
    dense = att.dense_decode(q, K, V, scale)
    assert np.all(np.isfinite(dense))
    s = scale * np.einsum("hd,nhd->hn", att.widen(q), np.repeat(att.widen(K), 4, axis=1))
    assert np.max(np.abs(s)) > qscale      # logits of order qscale (|s| ~ 1e3 at x1000)
    ref = _sdpa_f64(att.widen(q), att.widen(K), att.widen(V), scale)
    assert np.max(np.abs(dense - ref)) < 1e-12
    online = att.online_decode_blocks(q, K, V, scale, 16)
    assert np.max(np.abs(online - dense)) < 1e-12


# -- multi-token query --------------------------------------------------------
def _sdpa_causal_tail_f64(q, K, V, scale):
    """q [T, H_q, d] at the last T of n positions, K/V [n, H_kv, d] -> [T, H_q, d]
    through torch SDPA with an explicit bottom-right causal mask (n >= T)."""
    T, H_q, _ = q.shape
    n, H_kv, _ = K.shape
    G = H_q // H_kv
    qt = torch.from_numpy(q).permute(1, 0, 2)                               # [H_q, T, d]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, dim=0)   # [H_q, n, d]
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, dim=0)
    pos = torch.arange(n)[None, :]
    mask = pos <= (n - T + torch.arange(T))[:, None]                        # [T, n]
    out = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None],
                                                           attn_mask=mask, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("n,T,H_q,H_kv,d", [(9, 3, 8, 2, 16), (40, 4, 4, 4, 32), (5, 5, 2, 1, 8),
                                            (100, 8, 16, 8, 64), (17, 16, 1, 1, 16)])
def test_multi_query_matches_torch_causal_sdpa(n, T, H_q, H_kv, d):
    g = rng(300 + n + T)
    q = normal_f32(g, (T, H_q, d)).astype(np.float64)
    K = normal_f32(g, (n, H_kv, d)).astype(np.float64)
    V = normal_f32(g, (n, H_kv, d)).astype(np.float64)
    scale = 1.0 / np.sqrt(d)
    ref = _sdpa_causal_tail_f64(q, K, V, scale)
    out = att.multi_query(q, K, V, scale)
    assert np.max(np.abs(out - ref)) < 1e-13


def test_multi_query_special_cases():
    g = rng(7)
    T, H_q, H_kv, d = 4, 4, 2, 16
    q = normal_bf16_bits(g, (T, H_q, d))
    K = normal_bf16_bits(g, (6, H_kv, d))
    V = normal_bf16_bits(g, (6, H_kv, d))
    # one token: plain decode over the whole history
    one = att.multi_query(q[:1], K, V, 0.25)
    assert np.array_equal(one[0], att.dense_decode(q[0], K, V, 0.25))
    # the last token sees everything; token 0 of a history of T tokens sees only token 0 -> v_0
    out = att.multi_query(q, K[:T], V[:T], 0.25)
    assert np.array_equal(out[-1], att.dense_decode(q[-1], K[:T], V[:T], 0.25))
    Vf = att.widen(V)
    for h in range(H_q):
        assert np.array_equal(out[0, h], Vf[0, h // (H_q // H_kv)])
    # fewer tokens than queries: tokens before the history's start give 0
    short = att.multi_query(q, K[:2], V[:2], 0.25)
    assert not short[:2].any()
    assert np.array_equal(short[2, 0], Vf[0, 0])
    # causality: poisoning the positions after token i leaves row i unchanged
    Kp, Vp = att.widen(K).copy(), att.widen(V).copy()
    Kp[4:] = np.nan
    Vp[4:] = np.nan
    pois = att.multi_query(q, Kp, Vp, 0.25)
    clean = att.multi_query(q, K, V, 0.25)
    assert np.array_equal(pois[:2], clean[:2])      # tokens at positions 2, 3
    assert np.isnan(pois[2:]).all()


# -- per-head checker and the bf16 decoder -------------------------------------
# ``dense_decode_head`` is the checker of the full-size sampled parity tests and
# ``widen`` decodes every bf16 bit pattern on the oracle's side; both are pinned
# here against library routines and exact values, not against other oracle code.
def _sdpa_head_f64(q_h, K, V, scale):
    """q_h [d], K/V [n, d] float64 -> [d] via torch SDPA (one head)."""
    qt = torch.from_numpy(np.ascontiguousarray(q_h))[None, None, None, :]
    kt = torch.from_numpy(np.ascontiguousarray(K))[None, None]
    vt = torch.from_numpy(np.ascontiguousarray(V))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return out[0, 0, 0].numpy()


def _bf16_bits_to_f64_torch(bits):
    """bf16 bit patterns -> float64 through torch's own bfloat16 conversion on the CPU."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


@pytest.mark.parametrize("n,H_q,H_kv,d,kind,qscale",
                         [(1, 4, 1, 8, "f32", 1.0), (5, 8, 2, 16, "f32", 1.0), (37, 8, 2, 64, "bf16", 1.0),
                          (200, 32, 8, 128, "bf16", 1.0), (64, 32, 4, 128, "bf16", 1000.0),
                          (17, 16, 4, 32, "f32", 1000.0), (300, 8, 8, 128, "bf16", 30.0)])
def test_dense_decode_head_matches_sdpa(n, H_q, H_kv, d, kind, qscale):
    """Every (query head h, KV head h // G) through the per-head checker equals
    torch SDPA in float64 on the same widened values, for float32 and bf16 bit
    inputs, with logits up to |s| ~ 1e3."""
    g = rng(700 + n + d)
    draw = normal_f32 if kind == "f32" else normal_bf16_bits
    q = draw(g, (H_q, d), qscale)
    K = draw(g, (n, H_kv, d))
    V = draw(g, (n, H_kv, d))
    scale = 1.0 / np.sqrt(d)
    G = H_q // H_kv
    qf = q.astype(np.float64) if kind == "f32" else _bf16_bits_to_f64_torch(q)
    Kf = K.astype(np.float64) if kind == "f32" else _bf16_bits_to_f64_torch(K)
    Vf = V.astype(np.float64) if kind == "f32" else _bf16_bits_to_f64_torch(V)
    for h in range(H_q):
        out = att.dense_decode_head(q[h], K[:, h // G], V[:, h // G], scale)
        assert np.all(np.isfinite(out))
        ref = _sdpa_head_f64(qf[h], Kf[:, h // G], Vf[:, h // G], scale)
        assert np.max(np.abs(out - ref)) < 1e-12, (h, np.max(np.abs(out - ref)))


def test_dense_decode_head_special_cases():
    g = rng(71)
    d = 32
    # length 0 -> zeros of the head's width
    z = att.dense_decode_head(normal_f32(g, (d,)), np.zeros((0, d), np.float32), np.zeros((0, d), np.float32), 0.5)
    assert z.shape == (d,) and not z.any()
    # length 1 -> v_0 exactly (bf16 input)
    K1, V1 = normal_bf16_bits(g, (1, d)), normal_bf16_bits(g, (1, d))
    one = att.dense_decode_head(normal_bf16_bits(g, (d,)), K1, V1, 0.25)
    assert np.array_equal(one, _bf16_bits_to_f64_torch(V1)[0])
    # one dominant logit selects that token's value
    K = normal_f32(g, (40, d))
    V = normal_f32(g, (40, d))
    dom = att.dense_decode_head(K[23] * 1000.0, K, V, 1.0)
    np.testing.assert_allclose(dom, V[23].astype(np.float64), rtol=0, atol=1e-12)


def test_widen_matches_torch_bfloat16():
    """The bf16 decoder against torch's bfloat16 -> float64 conversion over every
    one of the 65,536 bit patterns (NaNs compared as NaN), and exact values."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):   # signalling-NaN patterns
        ours = att.widen(bits)
    ref = _bf16_bits_to_f64_torch(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))
    fixed = {0x3F80: 1.0, 0xC000: -2.0, 0x0000: 0.0, 0x4049: 3.140625, 0x3F00: 0.5,
             0x0001: 2.0 ** -133, 0x0080: 2.0 ** -126, 0x7F7F: (2.0 - 2.0 ** -7) * 2.0 ** 127,
             0x7F80: np.inf, 0xFF80: -np.inf}
    for b, v in fixed.items():
        assert att.widen(np.array([b], np.uint16))[0] == v, hex(b)
    neg0 = att.widen(np.array([0x8000], np.uint16))[0]
    assert neg0 == 0.0 and np.signbit(neg0)
    # float inputs pass through exactly
    x = normal_f32(rng(72), (100,))
    assert np.array_equal(att.widen(x), x.astype(np.float64))
