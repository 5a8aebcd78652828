"""Multi-token query paged attention on the GPU against the float64 oracle.

T query tokens per request sit at the last T positions of its history (their
K/V already in the pools) and attend causally: token i sees positions up to
seq_len - T + i.  The oracle is ``oracle.attention.multi_query``, pinned to
torch's causal SDPA on the CPU.  Tolerances as for single-token decode:
1e-5 for fp32 pools, 1e-2 for bf16 pools with an fp32 output.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
from tests.paged_batch import as_f64, device_batch, host_batch, torch_from_host

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 1e-2

EDGE_LENS = (0, 1, 2, 3, 4, 5, 15, 16, 17, 33, 100, 257, 1000)


@pytest.fixture(params=[0, 1, 2], ids=["auto", "fma", "mma"])
def kernel(request):
    import paged_kv_cache_358_b200 as pkv

    pkv.set_decode_kernel(request.param)
    yield request.param
    pkv.set_decode_kernel(0)


def _case(T, Hq, Hkv, D, B, dtype, lengths, seed):
    wl = W.DecodeWorkload(f"mq_T{T}", 1, Hq, Hkv, D, B, dtype, tuple(lengths),
                          pool_blocks=sum(-(-n // B) for n in lengths) + 8, seed=seed)
    hb = host_batch(wl)
    g = W.rng(seed + 1000)
    shape = (len(lengths), T, Hq, D)
    q = W.normal_bf16_bits(g, shape) if dtype == "bf16" else W.normal_f32(g, shape)
    return wl, hb, q


def _ref(hb, q):
    return np.stack([oatt.multi_query(q[s], hb.k_hist[s], hb.v_hist[s], hb.wl.scale)
                     for s in range(len(hb.lengths))])


@pytest.mark.parametrize("T,Hq,Hkv,D,B,dtype", [
    (2, 32, 8, 128, 16, "bf16"),   # 8 columns per KV head: tensor-core tiles
    (4, 32, 8, 128, 16, "bf16"),   # 16 columns: columns-in-M tensor-core tiles (CUDA-core when forced)
    (3, 8, 4, 64, 8, "bf16"),      # 6 columns padded to 8
    (5, 4, 4, 256, 32, "bf16"),    # 5 columns padded to 8, 512-byte rows
    (3, 16, 4, 64, 16, "f32"),     # 12 columns padded to 16, fp32 pools
    (16, 8, 8, 128, 4, "f32"),     # 16 tokens, no grouping, 4-token blocks
    (2, 6, 2, 128, 16, "bf16"),    # a group of 3: 6 columns padded to 8
    (4, 32, 8, 128, 4, "bf16"),    # 16 columns at block size 4: tiles laid out block by block
    (2, 16, 4, 128, 4, "bf16"),    # 8 columns at block size 4
])
def test_multi_query_all_outputs(kernel, T, Hq, Hkv, D, B, dtype):
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl, hb, q = _case(T, Hq, Hkv, D, B, dtype, EDGE_LENS, seed=40 + T)
    db = device_batch(hb)
    out = pkv.paged_attn_multi_query(torch_from_host(q), db.k_pool, db.v_pool, db.tables, db.seq_lens,
                                     wl.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    got = as_f64(out)
    ref = _ref(hb, q)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    assert err.max() <= tol, f"max err {err.max():.3e}"
    # tokens before the start of a short history attend nothing
    for s, n in enumerate(hb.lengths):
        for i in range(T):
            if n - T + i < 0:
                assert not got[s, i].any()


def test_multi_query_long_histories_bf16_out():
    """8 requests of 4096 tokens (split across many CTAs), T = 2, bf16 output."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl, hb, q = _case(2, 32, 8, 128, 16, "bf16", (4096,) * 8, seed=77)
    db = device_batch(hb)
    out = pkv.paged_attn_multi_query(torch_from_host(q), db.k_pool, db.v_pool, db.tables, db.seq_lens,
                                     wl.scale)
    torch.cuda.synchronize()
    got = as_f64(out)
    ref = _ref(hb, q)
    tol = TOL_BF16 + np.abs(ref) * 2.0 ** -8
    assert np.all(np.abs(got - ref) <= tol)


def test_single_token_equals_decode():
    """T = 1 through the multi-token entry is the decode kernel, bit for bit."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl, hb, q = _case(1, 32, 8, 128, 16, "bf16", EDGE_LENS, seed=5)
    db = device_batch(hb)
    qd = torch_from_host(q)
    a = pkv.paged_attn_multi_query(qd, db.k_pool, db.v_pool, db.tables, db.seq_lens, wl.scale,
                                   out_dtype=torch.float32)
    b = pkv.paged_decode_attn(qd[:, 0].contiguous(), db.k_pool, db.v_pool, db.tables, db.seq_lens, wl.scale,
                              out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a[:, 0], b)


def test_multi_query_rejects_unsupported_shapes():
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl, hb, q = _case(2, 32, 8, 128, 16, "bf16", (5, 9), seed=9)
    db = device_batch(hb)
    L = pkv.lib()
    for T in (0, 5, 17):  # 5 * 4 = 20 columns per KV head is more than 16
        assert L.pkv_multi_query_workspace_bytes(2, T, 32, 8, 128) == 0
        qq = torch.zeros((2, max(T, 1), 32, 128), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(qq)
        ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
        rc = L.pkv_paged_attn_multi_query(qq.data_ptr(), T, db.k_pool.data_ptr(), db.v_pool.data_ptr(),
                                          db.tables.data_ptr(), db.tables.shape[1], db.seq_lens.data_ptr(),
                                          2, 32, 8, 128, 16, wl.pool_blocks, wl.scale, pkv.BF16,
                                          out.data_ptr(), pkv.BF16, ws.data_ptr(), ws.numel(), None)
        assert rc == pkv.Status.INVALID


@pytest.mark.parametrize("T,Hq,Hkv", [
    (1, 32, 2),     # single token, 16 grouped heads: the split pieces merged by their own launch
    (4, 8, 2),      # 4 tokens of 4 heads: 16 columns, causal
    (2, 8, 2),      # 2 tokens of 4 heads: 8 columns, causal, also merged by their own launch
    (1, 12, 2),     # 6 heads padded to 8 columns: merged by their own launch
    (1, 8, 2),      # 4 columns: merged by the last CTA to finish a pair
])
def test_stale_workspace_bytes_never_reach_the_output(T, Hq, Hkv):
    """Fewer tiles than CTAs: most CTAs own no tile, so a split pair's pieces
    sit on CTAs with empty ones between them, whose partial-state slots are
    never written.  With the workspace filled with 0xFF bytes (NaN as fp32)
    before the call, the outputs must equal those of a zeroed workspace
    bit for bit, and the oracle's.  (The first word, the status that faults
    accumulate in until pkv_decode_status reads it, is read and cleared once
    after the fill; every other byte stays stale.)"""
    import torch

    import paged_kv_cache_358_b200 as pkv

    D, B = 128, 16
    lengths = (37, 91, 128, 201, 511, 0, 1, 17)
    wl, hb, q = _case(T, Hq, Hkv, D, B, "bf16", lengths, seed=90 + T)
    db = device_batch(hb)
    S = len(lengths)
    n = pkv.lib().pkv_multi_query_workspace_bytes(S, T, Hq, Hkv, D)
    outs = []
    for fill in (0x00, 0xFF):
        ws = torch.full((int(n),), fill, dtype=torch.uint8, device="cuda")
        pkv.decode_status(ws)
        outs.append(pkv.paged_attn_multi_query(torch_from_host(q), db.k_pool, db.v_pool, db.tables, db.seq_lens,
                                               wl.scale, out_dtype=torch.float32, workspace=ws))
        assert pkv.decode_status(ws) == pkv.Status.OK
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    got = as_f64(outs[1])
    assert np.all(np.isfinite(got))
    assert np.abs(got - _ref(hb, q)).max() <= TOL_BF16
